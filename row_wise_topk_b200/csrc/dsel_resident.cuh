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
// kernel reads it once into shared memory and selects there, exactly:
//
//   1. bulk copies of the row, one 4 KB chunk (one 16-byte vector per thread)
//      per mbarrier, so that step 2 starts on the first chunk;
//   2. each thread keeps the largest key of each of its vectors in a register,
//      and the CTA finds the row's largest and smallest keys and any NaN;
//   3. seed: when the row has at least k vectors, the k-th largest vector
//      maximum T0 is a lower bound of the k-th largest element (k vectors each
//      hold an element >= T0); a histogram of the vector maxima gives it;
//   4. the exact k-th largest key: histograms of the keys >= T0 in 1024 bins
//      spread over the remaining key range, one level per pass, until the
//      boundary bin is a single key or holds at most 128 elements, which are
//      then ranked directly;
//   5. output in index order without sorting: each vector's counts of keys
//      above the k-th key and equal to it, scanned over the row in index order,
//      give every selected element its output slot (equal keys are taken in
//      index order, the tie rule value-descending then index-ascending).
//
// Every pass tests a whole vector against its bound with packed compares and
// visits only the elements that pass, in rolled loops.  Histogram levels rotate
// over three buffers; the buffer of level L + 2 is cleared after the barrier of
// level L, when its last readers are done.  Value order and the sampling step
// put the k selected entries in shared memory instead and finish as the
// streaming kernel does (bitonic sort, draw).
#pragma once

#include "dsel_kernels.cuh"

namespace dsel {

constexpr int kResBins = 1024;
constexpr int kResVpt = kResRowBytes / (kResThreads * kVecBytes);   // vectors per thread: 8
static_assert(kResVpt == 8, "rows of up to 32 KB: 8 vectors per thread");
static_assert(kMaxK <= 4096 && kResRowBytes / 2 < (1 << 20), "output counts pack as 12 + 20 bits");

// Largest and smallest key of a 16-byte vector; true when it holds a NaN.
template <int DT>
__device__ __forceinline__ bool vec_minmax_key(const uint4 x, uint32_t& kmx, uint32_t& kmn) {
  using E = Elem<DT>;
  if (DT == DSEL_BF16) {
    const uint32_t hi = bf16x2_max_nan(bf16x2_max_nan(x.x, x.y), bf16x2_max_nan(x.z, x.w));
    const uint32_t lo = bf16x2_min_nan(bf16x2_min_nan(x.x, x.y), bf16x2_min_nan(x.z, x.w));
    if (E::is_nan(hi & 0xFFFFu) || E::is_nan(hi >> 16)) return true;
    kmx = max(E::key(hi & 0xFFFFu), E::key(hi >> 16));
    kmn = min(E::key(lo & 0xFFFFu), E::key(lo >> 16));
    return false;
  } else {
    const float a = __uint_as_float(x.x), b = __uint_as_float(x.y), c = __uint_as_float(x.z),
                d = __uint_as_float(x.w);
    const float hi = f32_max_nan(f32_max_nan(a, b), f32_max_nan(c, d));
    const float lo = f32_min_nan(f32_min_nan(a, b), f32_min_nan(c, d));
    if (hi != hi) return true;
    kmx = E::key(__float_as_uint(hi));
    kmn = E::key(__float_as_uint(lo));
    return false;
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
  constexpr int NE = VPT * NW;         // scan-table entries
  constexpr int EPL = (NE + 31) / 32;  // of them per lane
  static_assert(VPT <= 32, "one bit per round");

  extern __shared__ __align__(1024) unsigned char smem[];
  const unsigned char* rowb = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.off_bars);
  int* hist = reinterpret_cast<int*>(smem + p.off_hist);            // 3 x kResBins
  uint32_t* tab = reinterpret_cast<uint32_t*>(smem + p.off_tab);    // [VPT][NW] packed warp totals
  uint32_t* offw = tab + NE;                                         // [NW][VPT] packed offsets
  bits_t* cb = reinterpret_cast<bits_t*>(smem + p.off_cb);
  uint32_t* ci = reinterpret_cast<uint32_t*>(smem + p.off_ci);
  Ctl& ctl = *reinterpret_cast<Ctl*>(smem + p.off_ctl);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t row = blockIdx.x;
  const int k = p.k;

#pragma unroll 1
  for (int i = tid; i < 3 * kResBins / 4; i += T) reinterpret_cast<int4*>(hist)[i] = make_int4(0, 0, 0, 0);
  if (tid == 0) {
    ctl.nan_found = 0;
    ctl.abort = 0;
    ctl.tie_n = 0;
    ctl.r_kmax = 0u;
    ctl.r_kmin = 0xFFFFFFFFu;
    ctl.r_gmin = 0xFFFFFFFFu;
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

  // ---- 2. vector maxima, row extremes, NaN ----
  uint32_t gk[VPT];   // largest key of vector i * T + tid; 0 = no vector (keys of numbers are >= 1)
  uint32_t kmax = 0u, kmin = 0xFFFFFFFFu, gmin = 0xFFFFFFFFu;
  bool nan = false, late = false;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    gk[i] = 0u;
    if (i < nch) {
      if (!mbar_wait(smem_u32(&bars[i]), 0u)) late = true;
      const int v = i * T + tid;
      if (v < nvec) {
        const uint4 x = *reinterpret_cast<const uint4*>(rowb + v * kVecBytes);
        const int valid = min(PV, n - v * PV);
        uint32_t mx = 0u, mn = 0xFFFFFFFFu;
        bool vn = false;
        if (valid == PV) {
          vn = vec_minmax_key<DT>(x, mx, mn);
        } else {
#pragma unroll 1
          for (int e = 0; e < valid; ++e) {
            const uint32_t b = vec_elem_dyn<DT>(x, e);
            if (E::is_nan(b)) vn = true;
            const uint32_t kk = E::key(b);
            mx = max(mx, kk);
            mn = min(mn, kk);
          }
        }
        if (vn) {
          nan = true;
        } else {
          gk[i] = mx;
          kmax = max(kmax, mx);
          kmin = min(kmin, mn);
          gmin = min(gmin, mx);
        }
      }
    }
  }
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  gmin = __reduce_min_sync(0xffffffffu, gmin);
  const bool wnan = __any_sync(0xffffffffu, nan), wlate = __any_sync(0xffffffffu, late);
  if (lane == 0) {
    atomicMax(&ctl.r_kmax, kmax);
    atomicMin(&ctl.r_kmin, kmin);
    atomicMin(&ctl.r_gmin, gmin);
    if (wnan) ctl.nan_found = 1;
    if (wlate) ctl.abort = 1;
  }
  __syncthreads();
  if (ctl.abort) {   // a copy may still be in flight: wait for it (bounded) before the CTA exits
    if (tid < nch) mbar_wait(smem_u32(&bars[tid]), 0u);
    return;
  }
  grid_launch_dependents();   // the row is in shared memory: the next launch may start its prologue
  if (ctl.nan_found) {
    if (!p.nan_flag) nan_trap();   // the pages' default NaN policy
    write_sentinel_row<DT, T>(p, row, DSEL_IDX_NAN);
    return;
  }
  kmax = ctl.r_kmax;
  kmin = ctl.r_kmin;
  gmin = ctl.r_gmin;

  // ---- 3. seed: the k-th largest vector maximum (or a bin edge below it) ----
  uint32_t lo = kmin, hi = kmax;   // the k-th largest key lies in [lo, hi]
  int above = 0;                   // elements with key > hi
  if (nvec >= k) {
    // bins 16 times narrower than [gmin, kmax] needs, the last one open below: the
    // top sixteenth of the range, where the k-th largest maximum usually lies, at
    // fine resolution
    const int s = max(0, res_shift(kmax - gmin) - 4);
#pragma unroll
    for (int i = 0; i < VPT; ++i)
      if (gk[i] != 0u) atomicAdd(&hist[min((kmax - gk[i]) >> s, static_cast<uint32_t>(kResBins - 1))], 1);
    __syncthreads();
    const BinHit bh = res_find_bin(hist, k, lane);
    lo = max(lo, bh.bin == kResBins - 1 ? gmin : res_bin_lo(kmax, gmin, bh.bin, s));
  }

  // Rounds whose vector (this thread's) has a key >= t: one bit per round.  The
  // passes below loop over these bits, and over the passing elements of each
  // vector, in rolled loops (small code: the instruction cache holds it).
  auto rounds_ge = [&](uint32_t t) -> uint32_t {
    uint32_t r = 0u;
#pragma unroll
    for (int i = 0; i < VPT; ++i) r |= gk[i] >= t ? (1u << i) : 0u;
    return r;
  };

  // ---- 4. the exact k-th largest key: histogram levels over [lo, hi] ----
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

  // ---- 5. output slots in index order ----
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

}  // namespace dsel
