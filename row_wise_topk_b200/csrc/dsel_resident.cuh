// Row-resident TopK: one CTA of 256 threads per row holds the whole row (at most
// 32 KB: 16,384 bf16 or 8,192 f32 elements) in shared memory.
//
// The streaming kernel (topk_stream_kernel) follows the method of "DeepSeek
// releases DeepSelect, a TopK kernel for sparse attention and sampling" (method
// paragraph): a threshold filter over blocks read once, a candidate buffer, and
// radix-select compactions.  Its fixed cost per row (seed histogram, exact test,
// final select, index ranking, each behind several barriers) dominates when a
// row is only a few thousand elements, as in a batch of variable-length indexer
// rows.  Such a row fits in shared memory next to everything else, so this
// kernel reads it once into shared memory and selects there, exactly, with the
// same threshold filter made dense:
//
//   1. bulk copies of the row, one 4 KB chunk (one 16-byte vector per thread)
//      per mbarrier, so that step 2 starts on the first chunk;
//   2. each thread keeps the largest key of each of its vectors in a register;
//      the CTA finds the row's largest key and any NaN;
//   3. the threshold T0: at least k elements are >= T0.  With at least k
//      vectors it is the lower edge of the histogram bin holding the k-th
//      largest vector maximum (k vectors each hold an element >= T0); shorter
//      rows histogram their elements instead;
//   4. the vectors whose maximum reaches T0, listed in index order (one ballot
//      per vector slot, a prefix over the (round, warp) counts);
//   5. their elements >= T0: warp w expands the w-th part of that list into its
//      own list of row indices, so the warps' lists, one after the other, are
//      the candidates in index order;
//   6. the boundary: histograms of the candidates' keys in 1024 bins spread over
//      [T0, largest key], one level per pass, until the boundary bin is one key,
//      is taken whole, or holds at most 32 candidates, which are ranked directly;
//   7. output in index order: per-warp counts of the candidates above the
//      boundary and equal to it give every warp its first output slot; inside a
//      warp, ballots give the rest.  Equal keys are taken in index order (the
//      tie rule: value descending, then index ascending).
//
// A candidate list that overflows its share of shared memory (rows of very many
// equal keys) sends the row to resident_exact, which selects on the resident row
// itself: histogram levels over the vectors, then per-vector counts scanned in
// index order.  Value order and the sampling step put the k selected entries in
// shared memory instead and finish as the streaming kernel does (bitonic sort,
// draw).
#pragma once

#include "dsel_kernels.cuh"

namespace dsel {

constexpr int kResBins = 1024;
constexpr int kResVpt = kResRowBytes / (kResThreads * kVecBytes);   // vectors per thread: 8
constexpr int kResMembers = 32;   // a boundary bin of at most this many candidates is ranked directly
static_assert(kResVpt == 8, "rows of up to 32 KB: 8 vectors per thread");
static_assert(kMaxK <= 4096 && kResRowBytes / 2 < (1 << 20), "output counts pack as 12 + 20 bits");
static_assert(kResRowBytes / 2 <= 65536, "row indices fit 16 bits");

// Control block of the row-resident kernel.
struct __align__(16) ResCtl {
  float smp_w[kWarpsMax];       // sampling step: per-warp weight sums,
  int smp_c, smp_pos;           //   last kept candidate, drawn candidate,
  float smp_ec;                 //   weight sum of the kept candidates
  int flags;                    // bit 0: NaN seen, bit 1: a candidate list overflowed, bit 2: a wait gave up
  uint32_t kmax;                // the row's largest key
  uint32_t lmin;                // one less than its smallest vector maximum (rows of >= k vectors), else
                                //   than its smallest key
  uint32_t t0;                  // the candidate threshold
  int bin, before, cnt;         // a bin search, broadcast to the CTA
  int tie_n;                    // members of a small boundary bin gathered so far
  uint32_t r_tkey;              // the boundary key found by ranking,
  int r_ngt;                    //   and how many entries exceed it
  int w_a[kWarpsMax];           // per-warp counts: candidates above the boundary,
  int w_b[kWarpsMax];           //   and equal to it
  int vtab[kResVpt * (kResThreads / 32)];   // candidate vectors per (round, warp)
  uint32_t m_key[kResMembers];  // keys of a small boundary bin's members
};
static_assert(sizeof(ResCtl) <= kResCtlBytes, "row-resident control block outgrew its reservation");

// Largest key of a whole vector, without a NaN test: NaN-propagating packed
// maxima, folded into the thread's running accumulator `nacc`, which is tested once
// at the end (a row with a NaN is flagged whole, so the key of a vector holding
// one is never used).
template <int DT>
__device__ __forceinline__ uint32_t vec_max_key_fast(const uint4& x, uint32_t& nacc) {
  using E = Elem<DT>;
  if (DT == DSEL_BF16) {
    const uint32_t m2 = bf16x2_max_nan(bf16x2_max_nan(x.x, x.y), bf16x2_max_nan(x.z, x.w));
    nacc = bf16x2_max_nan(nacc, m2);
    const uint32_t m1 = bf16x2_max_nan(m2, __byte_perm(m2, 0u, 0x1032u));   // both halves: the larger
    return E::key(m1 & 0xFFFFu);
  } else {
    const float m = f32_max_nan(f32_max_nan(__uint_as_float(x.x), __uint_as_float(x.y)),
                                f32_max_nan(__uint_as_float(x.z), __uint_as_float(x.w)));
    nacc = __float_as_uint(f32_max_nan(__uint_as_float(nacc), m));
    return E::key(__float_as_uint(m));
  }
}

// True when the accumulator of vec_max_key_fast saw a NaN.
template <int DT>
__device__ __forceinline__ bool nacc_is_nan(uint32_t nacc) {
  using E = Elem<DT>;
  return DT == DSEL_BF16 ? (E::is_nan(nacc & 0xFFFFu) || E::is_nan(nacc >> 16)) : E::is_nan(nacc);
}

// Smallest key of a whole vector that holds no NaN (with a NaN the result is
// meaningless; such rows are flagged whole).
template <int DT>
__device__ __forceinline__ uint32_t vec_min_key(const uint4& x) {
  using E = Elem<DT>;
  if (DT == DSEL_BF16) {
    const uint32_t m2 = bf16x2_min_nan(bf16x2_min_nan(x.x, x.y), bf16x2_min_nan(x.z, x.w));
    return min(E::key(m2 & 0xFFFFu), E::key(m2 >> 16));
  } else {
    const float m = f32_min_nan(f32_min_nan(__uint_as_float(x.x), __uint_as_float(x.y)),
                                f32_min_nan(__uint_as_float(x.z), __uint_as_float(x.w)));
    return E::key(__float_as_uint(m));
  }
}

// Shift that spreads the key range [lo, lo + range] over at most 1024 bins.
__device__ __forceinline__ int res_shift(uint32_t range) { return max(0, (32 - __clz(range)) - 10); }

// Lowest key of bin b (bins of 2^s keys counted down from hi), not below lo.
__device__ __forceinline__ uint32_t res_bin_lo(uint32_t hi, uint32_t lo, int b, int s) {
  const uint64_t span = (static_cast<uint64_t>(b) + 1u) << s;   // keys from hi down to the bin's end
  return span > static_cast<uint64_t>(hi - lo) ? lo : hi - static_cast<uint32_t>(span) + 1u;
}

struct BinHit {
  int bin;      // the bin holding the t-th largest entry (bin 0 = the top)
  int before;   // entries in the bins above it
  int cnt;      // entries in it
};

// Bin of the t-th largest entry in a 1024-bin histogram (bin 0 = largest keys),
// found by one warp with no barrier; every warp may run it on the same
// histogram.  The histogram must hold at least t entries.
__device__ __forceinline__ BinHit res_find_bin(const int* h, int t, int lane) {
  const int sum = chunk_sum4<8>(reinterpret_cast<const int4*>(h), 0, lane);   // bins 32*lane .. +31
  const int incl = warp_incl_scan(sum, lane);
  const int L = max(0, __ffs(__ballot_sync(0xffffffffu, incl >= t)) - 1);
  const int base = __shfl_sync(0xffffffffu, incl - sum, L);
  const int c = h[32 * L + lane];
  const int incl2 = warp_incl_scan(c, lane) + base;
  const int j = max(0, __ffs(__ballot_sync(0xffffffffu, incl2 >= t)) - 1);
  BinHit res;
  res.bin = 32 * L + j;
  res.cnt = __shfl_sync(0xffffffffu, c, j);
  res.before = __shfl_sync(0xffffffffu, incl2, j) - res.cnt;
  return res;
}

// Bit e set when element e of the vector is valid (e < valid) and its key is
// >= t: one packed float compare against t's value per element pair (no NaN is
// left when this runs, and -0 and +0 compare equal as floats and as keys).
template <int DT>
__device__ __forceinline__ uint32_t res_mask_ge(const uint4& x, uint32_t t, int valid) {
  using E = Elem<DT>;
  const uint32_t b = E::bits_of_key(t);
  const uint32_t m = candidate_mask<DT>(x, DT == DSEL_BF16 ? (b | (b << 16)) : b);
  return valid >= E::kPerVec ? m : (m & ((1u << valid) - 1u));
}

// Exact selection on the resident row itself, for rows whose candidates did not
// fit their lists: every key of the row is >= lo or below the k-th largest key,
// and none exceeds kmax; no NaN.  Histogram levels over the keys in [lo, hi],
// restricted to the vectors whose maximum reaches lo, narrow [lo, hi] down to
// the k-th largest key (or a bin of at most 128 keys, ranked directly); then each
// vector's counts of keys above it and equal to it, scanned over the row in
// index order, give every selected element its output slot.  Histogram levels
// rotate over three buffers (the two histograms and the list space after them);
// the buffer of level L + 2 is cleared after the barrier of level L.
template <int DT>
__device__ __noinline__ void resident_exact(const KParams& p, unsigned char* smem, int64_t row, int n,
                                            uint32_t lo, uint32_t kmax) {
  using E = Elem<DT>;
  using bits_t = typename E::bits_t;
  constexpr int T = kResThreads;
  constexpr int VPT = kResVpt;
  constexpr int NW = T / 32;
  constexpr int PV = E::kPerVec;
  constexpr int CH = T * kVecBytes;
  constexpr int NE = VPT * NW;         // scan-table entries
  constexpr int EPL = (NE + 31) / 32;  // of them per lane
  static_assert(VPT <= 32, "one bit per round");
  const unsigned char* rowb = smem;
  int* hist = reinterpret_cast<int*>(smem + p.off_hist);            // 3 x kResBins
  uint32_t* tab = reinterpret_cast<uint32_t*>(smem + p.off_tab);    // [VPT][NW] packed warp totals
  uint32_t* offw = tab + NE;                                         // [NW][VPT] packed offsets
  bits_t* cb = reinterpret_cast<bits_t*>(smem + p.off_cb);
  uint32_t* ci = reinterpret_cast<uint32_t*>(smem + p.off_ci);
  ResCtl& ctl = *reinterpret_cast<ResCtl*>(smem + p.off_ctl);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int k = p.k;
  const int nvec = (n + PV - 1) / PV;
  const uint32_t bytes = static_cast<uint32_t>((n + 15) / 16 * 16) * E::kBytes;
  const int nch = static_cast<int>((bytes + CH - 1) / CH);

#pragma unroll 1
  for (int i = tid; i < 3 * kResBins / 4; i += T) reinterpret_cast<int4*>(hist)[i] = make_int4(0, 0, 0, 0);
  uint32_t gk[VPT];   // largest key of vector i * T + tid; 0 = no vector (keys of numbers are >= 1)
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    gk[i] = 0u;
    const int v = i * T + tid;
    if (i < nch && v < nvec) {
      const uint4 x = *reinterpret_cast<const uint4*>(rowb + v * kVecBytes);
      const int valid = min(PV, n - v * PV);
      uint32_t mx = 0u;
#pragma unroll 1
      for (int e = 0; e < valid; ++e) mx = max(mx, E::key(vec_elem_dyn<DT>(x, e)));
      gk[i] = mx;
    }
  }
  __syncthreads();

  // Rounds whose vector (this thread's) has a key >= t: one bit per round.
  auto rounds_ge = [&](uint32_t t) -> uint32_t {
    uint32_t r = 0u;
#pragma unroll
    for (int i = 0; i < VPT; ++i) r |= gk[i] >= t ? (1u << i) : 0u;
    return r;
  };

  // ---- the exact k-th largest key: histogram levels over [lo, hi] ----
  uint32_t hi = kmax;
  int above = 0;   // elements with key > hi
  uint32_t tkey;   // the k-th largest key
  int n_gt;        // elements with key > tkey (< k)
#pragma unroll 1
  for (int level = 1;; ++level) {
    int* h = hist + (level % 3) * kResBins;
    const int s = res_shift(hi - lo);
    uint32_t rm = rounds_ge(lo);   // only vectors whose maximum reaches lo hold such keys
#pragma unroll 1
    while (rm != 0u) {
      const int i = __ffs(rm) - 1;
      rm &= rm - 1u;
      const int v = i * T + tid;
      const uint4 x = *reinterpret_cast<const uint4*>(rowb + v * kVecBytes);
      uint32_t m = res_mask_ge<DT>(x, lo, n - v * PV);
#pragma unroll 1
      while (m != 0u) {
        const int e = __ffs(m) - 1;
        m &= m - 1u;
        const uint32_t kk = E::key(vec_elem_dyn<DT>(x, e));
        if (kk <= hi) atomicAdd(&h[(hi - kk) >> s], 1);
      }
    }
    __syncthreads();
    const BinHit bh = res_find_bin(h, k - above, lane);
    const uint32_t bhi = hi - (static_cast<uint32_t>(bh.bin) << s);
    const uint32_t blo = res_bin_lo(hi, lo, bh.bin, s);
    above += bh.before;
    if (s == 0) {   // the boundary bin is one key
      tkey = bhi;
      n_gt = above;
      break;
    }
    if (bh.cnt <= kTieMax) {
      // rank the boundary bin's members by key; the free buffer of level + 1 holds them
      uint32_t* lst = reinterpret_cast<uint32_t*>(hist + ((level + 1) % 3) * kResBins);
      uint32_t rb = rounds_ge(blo);
#pragma unroll 1
      while (rb != 0u) {
        const int i = __ffs(rb) - 1;
        rb &= rb - 1u;
        const int v = i * T + tid;
        const uint4 x = *reinterpret_cast<const uint4*>(rowb + v * kVecBytes);
        uint32_t m = res_mask_ge<DT>(x, blo, n - v * PV);
#pragma unroll 1
        while (m != 0u) {
          const int e = __ffs(m) - 1;
          m &= m - 1u;
          const uint32_t kk = E::key(vec_elem_dyn<DT>(x, e));
          if (kk <= bhi) {
            const int pos = atomicAdd(&ctl.tie_n, 1);
            if (pos < kResBins) lst[pos] = kk;
          }
        }
      }
      __syncthreads();
      const int need = k - above;
      if (tid < bh.cnt) {
        const uint32_t kj = lst[tid];
        int gt = 0, eq = 0;
#pragma unroll 4
        for (int i = 0; i < bh.cnt; ++i) {
          const uint32_t ki = lst[i];
          gt += ki > kj ? 1 : 0;
          eq += ki == kj ? 1 : 0;
        }
        if (gt < need && need <= gt + eq) {   // the need-th largest member
          ctl.r_tkey = kj;
          ctl.r_ngt = above + gt;
        }
      }
      __syncthreads();
      tkey = ctl.r_tkey;
      n_gt = ctl.r_ngt;
      break;
    }
    // another level over the boundary bin; clear the buffer of level + 2
    int4* z = reinterpret_cast<int4*>(hist + ((level + 2) % 3) * kResBins);
#pragma unroll 1
    for (int i = tid; i < kResBins / 4; i += T) z[i] = make_int4(0, 0, 0, 0);
    lo = blo;
    hi = bhi;
  }

  // ---- output slots in index order ----
  // per vector: (keys > tkey) | (keys == tkey) << 12, scanned over the row in
  // vector order (round, thread).  Fewer than k <= 4096 keys exceed tkey, so
  // every prefix of the first field fits its 12 bits; the second counts at most
  // the row's 16,384 elements.  Both come from two packed compares (keys >= tkey,
  // keys >= tkey + 1; no key exceeds kmax).
  const int need_eq = k - n_gt;
  const uint32_t rt = rounds_ge(tkey);
  auto vec_count = [&](int i) -> uint32_t {
    const int v = i * T + tid;
    const uint4 x = *reinterpret_cast<const uint4*>(rowb + v * kVecBytes);
    const uint32_t ge = __popc(res_mask_ge<DT>(x, tkey, n - v * PV));
    const uint32_t gt = tkey < kmax ? __popc(res_mask_ge<DT>(x, tkey + 1u, n - v * PV)) : 0u;
    return gt | ((ge - gt) << 12);
  };
  // this thread's counts per round, one byte each (greater | equal << 4, both <= 8):
  // rounds 0-3 in cnt_lo, 4-7 in cnt_hi, for the write pass
  static_assert(VPT <= 8 && PV <= 8, "a round's counts fit one byte");
  uint32_t cnt_lo = 0u, cnt_hi = 0u;
#pragma unroll 1
  for (int i = 0; i < nch; ++i) {   // warp totals per round
    const bool mine = (rt >> i) & 1u;
    uint32_t w = 0u;
    if (__any_sync(0xffffffffu, mine)) {
      const uint32_t c = mine ? vec_count(i) : 0u;
      w = __reduce_add_sync(0xffffffffu, c);
      const uint32_t byte = (c & 0xFu) | ((c >> 12) << 4);
      if (i < 4) cnt_lo |= byte << (8 * i);
      else cnt_hi |= byte << (8 * (i - 4));
    }
    if (lane == 0) tab[i * NW + warp] = w;
  }
  __syncthreads();
  const bool to_smem = p.order == DSEL_ORDER_VALUE || p.token_out != nullptr;
  {   // every warp: exclusive prefix of the [round][warp] totals; keep this warp's column
    const int ne = nch * NW;
    uint32_t t4[EPL], run = 0u;
#pragma unroll
    for (int j = 0; j < EPL; ++j) {
      const int e = EPL * lane + j;
      t4[j] = run;
      run += e < ne ? tab[e] : 0u;
    }
    uint32_t incl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const uint32_t b0 = incl - run;
#pragma unroll
    for (int j = 0; j < EPL; ++j) {
      const int e = EPL * lane + j;
      if (e < ne && e % NW == warp) offw[warp * VPT + e / NW] = b0 + t4[j];
    }
    __syncwarp();
  }
  const int64_t obase = row * static_cast<int64_t>(k);
#pragma unroll 1
  for (int i = 0; i < nch; ++i) {
    const bool mine = (rt >> i) & 1u;
    if (!__any_sync(0xffffffffu, mine)) continue;   // warp-uniform
    const uint32_t byte = ((i < 4 ? cnt_lo : cnt_hi) >> (8 * (i & 3))) & 0xFFu;
    const uint32_t c = (byte & 0xFu) | ((byte >> 4) << 12);
    uint32_t incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (c == 0u) continue;
    const uint32_t pre = offw[warp * VPT + i] + incl - c;
    int gtb = static_cast<int>(pre & 0xFFFu), eqb = static_cast<int>(pre >> 12);
    const int v = i * T + tid;
    const uint4 x = *reinterpret_cast<const uint4*>(rowb + v * kVecBytes);
    uint32_t m = res_mask_ge<DT>(x, tkey, n - v * PV);
#pragma unroll 1
    while (m != 0u) {   // ascending element order: index order
      const int e = __ffs(m) - 1;
      m &= m - 1u;
      const uint32_t b = vec_elem_dyn<DT>(x, e);
      const bool gt = E::key(b) > tkey;
      if (gt || eqb < need_eq) {
        const int pos = gtb + min(eqb, need_eq);
        const uint32_t idx = static_cast<uint32_t>(v * PV + e);
        if (pos < k) {
          if (to_smem) {
            cb[pos] = static_cast<bits_t>(b);
            ci[pos] = idx;
          } else {
            if (p.index_i64) static_cast<int64_t*>(p.indices_out)[obase + pos] = static_cast<int64_t>(idx);
            else static_cast<int32_t*>(p.indices_out)[obase + pos] = static_cast<int32_t>(idx);
            if (p.return_value) static_cast<bits_t*>(p.values_out)[obase + pos] = static_cast<bits_t>(b);
          }
        }
      }
      if (gt) ++gtb;
      else ++eqb;
    }
  }
  if (!to_smem) return;
  __syncthreads();
  bitonic_sort<DT, T, true>(cb, ci, k);
  write_rows_out<DT, T>(p, row, 0, k, cb, ci);
  if (DT == DSEL_F32 && p.token_out != nullptr)
    sample_draw<T>(p, row, reinterpret_cast<const uint32_t*>(cb), ci, k, ctl);
}

// One CTA per row (blockIdx.x).
template <int DT>
__global__ void __launch_bounds__(kResThreads, 4) topk_resident_kernel(const __grid_constant__ KParams p) {
  using E = Elem<DT>;
  using bits_t = typename E::bits_t;
  constexpr int T = kResThreads;
  constexpr int VPT = kResVpt;
  constexpr int NW = T / 32;
  constexpr int PV = E::kPerVec;
  constexpr int CH = T * kVecBytes;    // bytes per chunk: one vector per thread
  static_assert(NW % 2 == 0 && VPT * NW <= 64, "the (round, warp) table: two entries per lane");

  extern __shared__ __align__(1024) unsigned char smem[];
  const bits_t* rowe = reinterpret_cast<const bits_t*>(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.off_bars);
  int* h0 = reinterpret_cast<int*>(smem + p.off_hist);   // vector maxima (or keys), then odd levels
  int* h1 = h0 + kResBins;                                 // candidate keys, then even levels
  uint16_t* vl = reinterpret_cast<uint16_t*>(smem + p.off_tab);   // candidate vectors, index order
  bits_t* cb = reinterpret_cast<bits_t*>(smem + p.off_cb);
  uint32_t* ci = reinterpret_cast<uint32_t*>(smem + p.off_ci);
  ResCtl& ctl = *reinterpret_cast<ResCtl*>(smem + p.off_ctl);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t below = (1u << lane) - 1u;
  const int64_t row = blockIdx.x;
  const int k = p.k;
  const int seg = p.seg;
  uint16_t* el = reinterpret_cast<uint16_t*>(smem + p.off_cv) + warp * seg;   // this warp's candidates
  auto load_vec = [&](int v) -> uint4 { return *reinterpret_cast<const uint4*>(smem + v * kVecBytes); };

#pragma unroll 1
  for (int i = tid; i < 2 * kResBins / 4; i += T) reinterpret_cast<int4*>(h0)[i] = make_int4(0, 0, 0, 0);
  if (tid == 0) {
    ctl.flags = 0;
    ctl.kmax = 0u;
    ctl.lmin = 0xFFFFFFFFu;
    ctl.tie_n = 0;
  }
  if (tid < VPT) {
    mbar_init(smem_u32(&bars[tid]), 1);
    fence_mbar_init();
  }
  __syncthreads();
  // the set-up above touched shared memory only: it may overlap the previous launch
  grid_dependency_wait();
  bool bad_end;
  const int64_t n64 = row_length(p, row, &bad_end);
  if (bad_end || n64 <= k) {
    if (bad_end) write_sentinel_row<DT, T>(p, row, DSEL_IDX_BAD_END);
    else finish_short_row<DT, T>(p, row, n64, cb, ci, ctl);
    return;
  }
  const int n = static_cast<int>(n64);   // <= kResRowBytes / 2
  const int nvec = (n + PV - 1) / PV;
  const uint32_t bytes = static_cast<uint32_t>((n + 15) / 16 * 16) * E::kBytes;   // multiple of 16 B
  const int nch = static_cast<int>((bytes + CH - 1) / CH);                       // <= VPT

  // ---- 1. bulk copies: chunk c (vectors c*T .. c*T + T - 1) by lane c of warp 0 ----
  if (warp == 0 && lane < nch) {
    const uint32_t b = min(static_cast<uint32_t>(CH), bytes - static_cast<uint32_t>(lane) * CH);
    const uint32_t bar = smem_u32(&bars[lane]);
    mbar_expect_tx(bar, b);
    bulk_g2s(smem_u32(smem + lane * CH),
             static_cast<const char*>(p.x) + (row * p.row_stride) * E::kBytes + static_cast<int64_t>(lane) * CH, b,
             bar);
  }

  // ---- 2. vector maxima, the row's largest key, NaN; the smallest vector maximum
  //         (rows of at least k vectors) or the smallest key (shorter rows) ----
  const bool by_vec = nvec >= k;
  const int nfull = n / (T * PV);   // rounds whose vectors are all whole
  uint32_t gk[VPT];   // largest key of vector i * T + tid; 0 = no vector (keys of numbers are >= 1)
  uint32_t nacc = 0u;
  bool nan = false, late = false;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    gk[i] = 0u;
    if (i < nfull) {
      if (!mbar_wait(smem_u32(&bars[i]), 0u)) late = true;
      gk[i] = vec_max_key_fast<DT>(load_vec(i * T + tid), nacc);
    } else if (i < nch) {
      if (!mbar_wait(smem_u32(&bars[i]), 0u)) late = true;
      const int v = i * T + tid;
      if (v < nvec) {
        const uint4 x = load_vec(v);
        const int valid = n - v * PV;
        if (valid >= PV) {
          gk[i] = vec_max_key_fast<DT>(x, nacc);
        } else {   // the row's last vector, cut short
          uint32_t mx = 0u;
#pragma unroll 1
          for (int e = 0; e < valid; ++e) {
            const uint32_t b = vec_elem_dyn<DT>(x, e);
            nan |= E::is_nan(b);
            mx = max(mx, E::key(b));
          }
          gk[i] = mx;
        }
      }
    }
  }
  // kmax, and lmin - 1 (the row has at least one key, which is >= 1: the CTA
  // minimum does not wrap; a thread without vectors contributes 0 - 1 = 2^32 - 1)
  uint32_t kmax = 0u, lmin = 0xFFFFFFFFu;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    kmax = max(kmax, gk[i]);
    lmin = min(lmin, gk[i] - 1u);
  }
  if (!by_vec) {   // shorter rows: the smallest key instead
    lmin = 0xFFFFFFFFu;
#pragma unroll 1
    for (int i = 0; i < nch; ++i) {
      const int v = i * T + tid;
      if (v < nvec) {
        const uint4 x = load_vec(v);
        const int valid = n - v * PV;
        if (valid >= PV) {
          lmin = min(lmin, vec_min_key<DT>(x) - 1u);
        } else {
#pragma unroll 1
          for (int e = 0; e < valid; ++e) lmin = min(lmin, E::key(vec_elem_dyn<DT>(x, e)) - 1u);
        }
      }
    }
  }
  nan |= nacc_is_nan<DT>(nacc);
  {
    const int f = (__any_sync(0xffffffffu, nan) ? 1 : 0) | (__any_sync(0xffffffffu, late) ? 4 : 0);
    const uint32_t wk = __reduce_max_sync(0xffffffffu, kmax), wl = __reduce_min_sync(0xffffffffu, lmin);
    if (lane == 0) {
      atomicMax(&ctl.kmax, wk);
      atomicMin(&ctl.lmin, wl);
      if (f) atomicOr(&ctl.flags, f);
    }
  }
  __syncthreads();
  {
    const int f = ctl.flags;
    if (f & 4) {   // a copy may still be in flight: wait for it (bounded) before the CTA exits
      if (tid < nch) mbar_wait(smem_u32(&bars[tid]), 0u);
      return;
    }
    grid_launch_dependents();   // the row is in shared memory: the next launch may start its prologue
    if (f & 1) {
      if (!p.nan_flag) nan_trap();   // the pages' default NaN policy
      write_sentinel_row<DT, T>(p, row, DSEL_IDX_NAN);
      return;
    }
  }
  kmax = ctl.kmax;
  lmin = ctl.lmin + 1u;

  // ---- 3. the threshold T0: at least k elements are >= T0 ----
  if (by_vec) {
    // bins 16 times narrower than [lmin, kmax] needs, the last one open below: the
    // top sixteenth of the range, where the k-th largest maximum usually lies, at
    // fine resolution
    const int s = max(0, res_shift(kmax - lmin) - 4);
#pragma unroll
    for (int i = 0; i < VPT; ++i)
      if (gk[i] != 0u) atomicAdd(&h0[min((kmax - gk[i]) >> s, static_cast<uint32_t>(kResBins - 1))], 1);
    __syncthreads();
    if (warp == 0) {
      const BinHit bh = res_find_bin(h0, k, lane);
      if (lane == 0) ctl.t0 = bh.bin == kResBins - 1 ? lmin : res_bin_lo(kmax, lmin, bh.bin, s);
    }
  } else {   // fewer vectors than k: a histogram of the elements themselves
    const int s = res_shift(kmax - lmin);
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int v = i * T + tid;
      if (i < nch && v < nvec) {
        const uint4 x = load_vec(v);
        const int valid = n - v * PV;
#pragma unroll
        for (int e = 0; e < PV; ++e)
          if (e < valid) atomicAdd(&h0[(kmax - E::key(vec_elem<DT>(x, e))) >> s], 1);
      }
    }
    __syncthreads();
    if (warp == 0) {
      const BinHit bh = res_find_bin(h0, k, lane);
      if (lane == 0) ctl.t0 = res_bin_lo(kmax, lmin, bh.bin, s);
    }
  }
  __syncthreads();
  const uint32_t t0 = ctl.t0;

  // ---- 4. the vectors whose maximum reaches T0, in index order: vector
  //         i * T + tid goes after the candidate vectors of every earlier
  //         (round, warp) and of the lower lanes ----
  int vcount;
  {
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      if (i < nch) {
        const unsigned bal = __ballot_sync(0xffffffffu, gk[i] >= t0);
        if (lane == 0) ctl.vtab[i * NW + warp] = __popc(bal);
      }
    }
    __syncthreads();
    // exclusive prefix over the (round, warp) entries, two per lane; entry
    // i * NW + warp has the parity of warp
    const int ne = nch * NW;
    const int c0 = 2 * lane < ne ? ctl.vtab[2 * lane] : 0;
    const int c1 = 2 * lane + 1 < ne ? ctl.vtab[2 * lane + 1] : 0;
    const int incl = warp_incl_scan(c0 + c1, lane);
    vcount = __shfl_sync(0xffffffffu, incl, 31);
    const int mine = incl - c1 - ((warp & 1) ? 0 : c0);
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      if (i < nch) {
        const bool cand = gk[i] >= t0;
        const unsigned bal = __ballot_sync(0xffffffffu, cand);
        const int off = __shfl_sync(0xffffffffu, mine, (i * NW + warp) >> 1);
        if (cand) vl[off + __popc(bal & below)] = static_cast<uint16_t>(i * T + tid);
      }
    }
  }
  __syncthreads();   // the vector list is complete

  // ---- 5. their elements >= T0: warp w expands the w-th part of the vector list
  //         into its own list of row indices (index order within and across
  //         warps); the level-0 histogram of their keys over [T0, kmax] ----
  const uint32_t tb = E::bits_of_key(t0);
  const uint32_t tv2 = DT == DSEL_BF16 ? (tb | (tb << 16)) : tb;   // T0 as packed element bits
  int wcnt;
  {
    const int v0 = vcount * warp / NW, v1 = vcount * (warp + 1) / NW;
    int wrun = 0;   // entries of this warp's list (warp-uniform)
#pragma unroll 1
    for (int j0 = v0; j0 < v1; j0 += 32) {
      const int j = j0 + lane;
      uint32_t m = 0u, v = 0u;
      if (j < v1) {
        v = vl[j];
        m = candidate_mask<DT>(load_vec(static_cast<int>(v)), tv2);
        const int valid = n - static_cast<int>(v) * PV;
        if (valid < PV) m &= (1u << valid) - 1u;
      }
      const int cnt = __popc(m);
      const int incl = warp_incl_scan(cnt, lane);
      const int tot = __shfl_sync(0xffffffffu, incl, 31);
      if (wrun + tot <= seg) {   // warp-uniform; past it the list has overflowed and stays unwritten
        uint16_t* dst = el + (wrun + incl - cnt);
        const uint32_t e0 = v * PV;
#pragma unroll 1
        while (m != 0u) {
          *dst++ = static_cast<uint16_t>(e0 + static_cast<uint32_t>(__ffs(m) - 1));
          m &= m - 1u;
        }
      }
      wrun += tot;
    }
    wcnt = wrun <= seg ? wrun : 0;   // an overflowed list is incomplete: the fallback takes the row
    if (lane == 0 && wrun > seg) atomicOr(&ctl.flags, 2);
  }
  __syncwarp();   // the warp's list is visible to all its lanes
  auto key_of = [&](int j) -> uint32_t { return E::key(rowe[el[j]]); };
  uint32_t lo = t0, hi = kmax;
  int s = res_shift(hi - lo);
#pragma unroll 1
  for (int j = lane; j < wcnt; j += 32) atomicAdd(&h1[(hi - key_of(j)) >> s], 1);
  __syncthreads();   // lists, candidate histogram and overflow flag are final
  if (ctl.flags & 2) {   // uniform: select on the resident row instead
    resident_exact<DT>(p, smem, row, n, t0, kmax);
    return;
  }

  // ---- 6. the boundary: histogram levels over the candidates ----
  int need = k;        // entries still to take from [lo, hi]
  const int* h = h1;
  bool all_bin;        // the boundary bin is taken whole: every key >= kb
  uint32_t kb;         // else the boundary key: every key > kb, and `need` ties in index order
#pragma unroll 1
  for (int level = 0;; ++level) {
    if (warp == 0) {
      const BinHit bh = res_find_bin(h, need, lane);
      if (lane == 0) {
        ctl.bin = bh.bin;
        ctl.before = bh.before;
        ctl.cnt = bh.cnt;
      }
    }
    __syncthreads();
    const int bin = ctl.bin, cnt = ctl.cnt;
    need -= ctl.before;
    const uint32_t bhi = hi - (static_cast<uint32_t>(bin) << s);
    const uint32_t blo = res_bin_lo(hi, lo, bin, s);
    if (cnt == need || blo == bhi) {
      all_bin = cnt == need;
      kb = blo;
      break;
    }
    if (cnt <= kResMembers) {   // rank the bin's members directly
#pragma unroll 1
      for (int j = lane; j < wcnt; j += 32) {
        const uint32_t kk = key_of(j);
        if (kk >= blo && kk <= bhi) {
          const int q = atomicAdd(&ctl.tie_n, 1);
          if (q < kResMembers) ctl.m_key[q] = kk;
        }
      }
      __syncthreads();
      if (warp == 0) {
        const uint32_t kj = lane < cnt ? ctl.m_key[lane] : 0u;
        int gt = 0, eq = 0;
#pragma unroll 1
        for (int i = 0; i < cnt; ++i) {
          const uint32_t ki = __shfl_sync(0xffffffffu, kj, i);
          gt += ki > kj ? 1 : 0;
          eq += ki == kj ? 1 : 0;
        }
        if (lane < cnt && gt < need && need <= gt + eq) {   // the need-th largest member
          ctl.r_tkey = kj;
          ctl.r_ngt = gt;
        }
      }
      __syncthreads();
      kb = ctl.r_tkey;
      need -= ctl.r_ngt;
      all_bin = false;
      break;
    }
    lo = blo;
    hi = bhi;
    s = res_shift(hi - lo);
    // the next level's buffer was last read by the search before the previous barrier
    int* hn = (level & 1) ? h1 : h0;
#pragma unroll 1
    for (int i = tid; i < kResBins / 4; i += T) reinterpret_cast<int4*>(hn)[i] = make_int4(0, 0, 0, 0);
    __syncthreads();
#pragma unroll 1
    for (int j = lane; j < wcnt; j += 32) {
      const uint32_t kk = key_of(j);
      if (kk >= lo && kk <= hi) atomicAdd(&hn[(hi - kk) >> s], 1);
    }
    __syncthreads();
    h = hn;
  }

  // ---- 7. output slots in index order ----
  {   // per-warp counts; each entry keeps its kind in the index's two spare bits
      // (bit 15: above the boundary, bit 14: equal to it) for the write pass
    int na = 0, nt = 0;
#pragma unroll 1
    for (int j0 = 0; j0 < wcnt; j0 += 32) {
      const int j = j0 + lane;
      bool a = false, t = false;
      if (j < wcnt) {
        const uint32_t gi = el[j];
        const uint32_t kk = E::key(rowe[gi]);
        a = all_bin ? kk >= kb : kk > kb;
        t = !all_bin && kk == kb;
        el[j] = static_cast<uint16_t>(gi | (a ? 0x8000u : 0u) | (t ? 0x4000u : 0u));
      }
      na += __popc(__ballot_sync(0xffffffffu, a));
      nt += __popc(__ballot_sync(0xffffffffu, t));
    }
    if (lane == 0) {
      ctl.w_a[warp] = na;
      ctl.w_b[warp] = nt;
    }
  }
  __syncthreads();
  int total;
  int ra = warp_prefix_of<NW>(ctl.w_a, warp, lane, total);   // above-boundary entries of earlier warps
  int rt = warp_prefix_of<NW>(ctl.w_b, warp, lane, total);   // boundary-key entries of earlier warps
  const int my_ties = all_bin ? 0 : need;   // boundary-key entries taken, the first ones in index order
  const bool to_smem = p.order == DSEL_ORDER_VALUE || p.token_out != nullptr;
  const int64_t obase = row * static_cast<int64_t>(k);
  int32_t* o32 = static_cast<int32_t*>(p.indices_out) + obase;
  int64_t* o64 = static_cast<int64_t*>(p.indices_out) + obase;
  bits_t* ov = static_cast<bits_t*>(p.values_out) + obase;
  const int mode = to_smem ? 0 : (p.index_i64 ? 2 : 1) | (p.return_value ? 4 : 0);
#pragma unroll 1
  for (int j0 = 0; j0 < wcnt; j0 += 32) {   // the same entries per lane as the count pass
    const int j = j0 + lane;
    const uint32_t ent = j < wcnt ? el[j] : 0u;
    const bool a = ent & 0x8000u, t = ent & 0x4000u;
    const uint32_t gi = ent & 0x3FFFu;
    const unsigned am = __ballot_sync(0xffffffffu, a), tm = __ballot_sync(0xffffffffu, t);
    const int rank_t = rt + __popc(tm & below);   // boundary-key entries before this one
    if (a || (t && rank_t < my_ties)) {   // its slot: entries selected before it (fewer than k)
      const int pos = ra + __popc(am & below) + min(rank_t, my_ties);
      if (mode == 0) {
        cb[pos] = rowe[gi];
        ci[pos] = gi;
      } else {
        if (mode & 2) o64[pos] = static_cast<int64_t>(gi);
        else o32[pos] = static_cast<int32_t>(gi);
        if (mode & 4) ov[pos] = rowe[gi];
      }
    }
    ra += __popc(am);
    rt += __popc(tm);
  }
  if (!to_smem) return;
  __syncthreads();
  bitonic_sort<DT, T, true>(cb, ci, k);
  write_rows_out<DT, T>(p, row, 0, k, cb, ci);
  if (DT == DSEL_F32 && p.token_out != nullptr)
    sample_draw<T>(p, row, reinterpret_cast<const uint32_t*>(cb), ci, k, ctl);
}

}  // namespace dsel
