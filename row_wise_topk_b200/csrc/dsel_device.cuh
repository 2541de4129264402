// Device building blocks for the row-wise TopK kernels (sm_100a).
//
// Method ("DeepSeek releases DeepSelect, a TopK kernel for sparse attention and
// sampling", narracomm, method paragraph): a threshold T starts at -inf and only
// rises; the row is read once, in contiguous blocks of B elements visited in a
// random order; entries above T go to a candidate buffer in shared memory; when
// the buffer holds k + B2 entries a radix select cuts it back to exactly k and
// raises T to the k-th entry.
//
// Choices made here for B200:
//   * blocks move global -> shared memory with the bulk-copy (TMA) engine
//     (cp.async.bulk, completion on a per-stage mbarrier), many blocks in flight;
//   * T is a composite (key, index) so that "above T" respects the tie rule
//     (value descending, then index ascending) exactly, and a cheap float test
//     (max of a 16-byte vector >= T, unordered) screens vectors before the exact
//     test;  NaN fails every ordered compare, so the same test also catches NaN;
//   * rows are split into contiguous slices handled by the CTAs of a
//     thread-block cluster; CTAs share T through distributed shared memory and
//     run the final radix select on the sum of their histograms.
#pragma once

#include <cooperative_groups.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/dsel.h"

namespace cg = cooperative_groups;

namespace dsel {

constexpr uint64_t kWaitLimitNs = 2000000000ull;   // bounded waits: 2 s
#ifndef DSEL_SUSPEND_HINT_NS
#define DSEL_SUSPEND_HINT_NS 20000
#endif
constexpr uint32_t kSuspendHintNs = DSEL_SUSPEND_HINT_NS;   // a waiting warp sleeps (woken at completion); 0: no hint
constexpr int kDigitBits = 8;
constexpr int kTieMax = 128;                  // radix select: largest bucket finished by direct ranking
constexpr int kBins = 1 << kDigitBits;

__device__ int g_device_status;                    // DSEL_ERR_DEVICE_TIMEOUT when a wait gave up

// --------------------------------------------------------------------------- //
// Element traits: order-preserving keys.  Canonicalising -0 to +0 first makes
// the two zeros one key; for every other non-NaN pattern, a larger value gives
// a larger unsigned key (sign bit set -> invert all bits, else set the sign bit).
// --------------------------------------------------------------------------- //
template <int DT> struct Elem;

template <> struct Elem<DSEL_BF16> {
  using bits_t = uint16_t;
  static constexpr int kKeyBits = 16;
  static constexpr int kBytes = 2;
  static constexpr int kPerVec = 8;
  static constexpr uint32_t kQNaN = 0x7FC0u;
  static constexpr uint32_t kNegInf = 0xFF80u;
  __device__ __forceinline__ static uint32_t key(uint32_t b) {
    b = (b == 0x8000u) ? 0u : b;
    return (b & 0x8000u) ? (~b & 0xFFFFu) : (b | 0x8000u);
  }
  __device__ __forceinline__ static uint32_t bits_of_key(uint32_t k) {
    return (k & 0x8000u) ? (k & 0x7FFFu) : (~k & 0xFFFFu);
  }
  __device__ __forceinline__ static bool is_nan(uint32_t b) { return (b & 0x7FFFu) > 0x7F80u; }
};

template <> struct Elem<DSEL_F32> {
  using bits_t = uint32_t;
  static constexpr int kKeyBits = 32;
  static constexpr int kBytes = 4;
  static constexpr int kPerVec = 4;
  static constexpr uint32_t kQNaN = 0x7FC00000u;
  static constexpr uint32_t kNegInf = 0xFF800000u;
  __device__ __forceinline__ static uint32_t key(uint32_t b) {
    b = (b == 0x80000000u) ? 0u : b;
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
  }
  __device__ __forceinline__ static uint32_t bits_of_key(uint32_t k) {
    return (k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k;
  }
  __device__ __forceinline__ static bool is_nan(uint32_t b) {
    return (b & 0x7FFFFFFFu) > 0x7F800000u;
  }
};

// Element e of a 16-byte vector (e is a compile-time constant after unrolling).
template <int DT>
__device__ __forceinline__ uint32_t vec_elem(const uint4& v, int e) {
  uint32_t w = (DT == DSEL_BF16) ? ((e >> 1) == 0 ? v.x : (e >> 1) == 1 ? v.y : (e >> 1) == 2 ? v.z : v.w)
                                 : (e == 0 ? v.x : e == 1 ? v.y : e == 2 ? v.z : v.w);
  if (DT == DSEL_BF16) return (e & 1) ? (w >> 16) : (w & 0xFFFFu);
  return w;
}

// --------------------------------------------------------------------------- //
// Screening test: true when some element of the vector may rank above T or is
// NaN.  `tv` is the threshold's value bits (bf16 pattern duplicated in both
// halves, or the f32 pattern).  Unordered >= is true for NaN on either side,
// so the initial T (a NaN pattern: key 0) lets everything through.
// --------------------------------------------------------------------------- //
__device__ __forceinline__ uint32_t bf16x2_max_nan(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.NaN.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ bool bf16x2_any_geu(uint32_t a, uint32_t t) {
  uint32_t r;
  asm("{\n\t.reg .pred p, q;\n\t"
      "setp.geu.bf16x2 p|q, %1, %2;\n\t"
      "or.pred p, p, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r) : "r"(a), "r"(t));
  return r != 0u;
}

// Non-propagating maxima (a NaN operand loses to a number).
__device__ __forceinline__ uint32_t bf16x2_max(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ float f32_max_nan(float a, float b) {
  float d;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
  return d;
}

// NaN-propagating minima.
__device__ __forceinline__ uint32_t bf16x2_min_nan(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("min.NaN.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ float f32_min_nan(float a, float b) {
  float d;
  asm("min.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
  return d;
}

// Candidate mask of a vector: bit e set when element e is >= T as a float, or NaN
// (unordered compare).  A superset of the elements that can rank above T.
__device__ __forceinline__ uint32_t bf16x2_geu_mask(uint32_t a, uint32_t t) {
  uint32_t r;
  asm("{\n\t.reg .pred p, q;\n\t"
      "setp.geu.bf16x2 p|q, %1, %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t"
      "@q or.b32 %0, %0, 2;\n\t}"
      : "=r"(r) : "r"(a), "r"(t));
  return r;
}

template <int DT>
__device__ __forceinline__ uint32_t candidate_mask(const uint4& v, uint32_t tv) {
  if (DT == DSEL_BF16) {
    return bf16x2_geu_mask(v.x, tv) | (bf16x2_geu_mask(v.y, tv) << 2) | (bf16x2_geu_mask(v.z, tv) << 4) |
           (bf16x2_geu_mask(v.w, tv) << 6);
  } else {
    const float t = __uint_as_float(tv);
    return (!(__uint_as_float(v.x) < t) ? 1u : 0u) | (!(__uint_as_float(v.y) < t) ? 2u : 0u) |
           (!(__uint_as_float(v.z) < t) ? 4u : 0u) | (!(__uint_as_float(v.w) < t) ? 8u : 0u);
  }
}

// Element e (a run-time value) of a 16-byte vector, without local memory.
template <int DT>
__device__ __forceinline__ uint32_t vec_elem_dyn(const uint4& v, int e) {
  if (DT == DSEL_BF16) {
    const int wi = e >> 1;
    const uint32_t w = wi < 2 ? (wi == 0 ? v.x : v.y) : (wi == 2 ? v.z : v.w);
    return (w >> ((e & 1) * 16)) & 0xFFFFu;
  } else {
    return e < 2 ? (e == 0 ? v.x : v.y) : (e == 2 ? v.z : v.w);
  }
}

template <int DT>
__device__ __forceinline__ bool screen(const uint4& v, uint32_t tv) {
  if (DT == DSEL_BF16) {
    uint32_t m = bf16x2_max_nan(bf16x2_max_nan(v.x, v.y), bf16x2_max_nan(v.z, v.w));
    return bf16x2_any_geu(m, tv);
  } else {
    float m = f32_max_nan(f32_max_nan(__uint_as_float(v.x), __uint_as_float(v.y)),
                          f32_max_nan(__uint_as_float(v.z), __uint_as_float(v.w)));
    return !(m < __uint_as_float(tv));
  }
}

// --------------------------------------------------------------------------- //
// PTX wrappers: mbarrier + bulk copy + timers.
// --------------------------------------------------------------------------- //
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  if (kSuspendHintNs == 0u) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0u;
  }
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(kSuspendHintNs)
      : "memory");
  return ok != 0u;
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait on a stage barrier; false when the limit ran out.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_ns() - t0 > kWaitLimitNs) {
      atomicExch(&g_device_status, DSEL_ERR_DEVICE_TIMEOUT);
      return false;
    }
  }
  return true;
}

__device__ __forceinline__ void nan_trap() { asm volatile("trap;"); }

// Programmatic dependent launch.  wait: block until the grids this launch
// depends on have completed and their writes are visible (a no-op for a launch
// without the programmatic-serialization attribute); everything before it must
// not touch global memory.  launch_dependents: let the next launch in the stream
// start its own prologue (it still waits for this grid before touching memory).
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" :::); }

// --------------------------------------------------------------------------- //
// Shared control block (one per CTA, after the candidate arrays).
// --------------------------------------------------------------------------- //
constexpr int kWarpsMax = 32;

struct __align__(16) Ctl {
  unsigned long long t_w;       // threshold word raised by peers (atomicMax); own T lives in registers
  unsigned long long x_vlo, x_vhi;
  unsigned long long wv[kWarpsMax];   // per-warp radix-word maxima
  int nan_found;
  int abort;
  int hb;                       // index of a histogram that is all zero
  int x_cnt, x_nan, x_kept;     // exchanged with peers in the final phase
  int sel_flag;
  int add[3];                   // survivors appended per round (round r uses add[r % 3])
  int tie_n;                    // radix select: members of a small bucket gathered so far
  unsigned long long tie_v;     // radix select: the selected radix word of that bucket
  int wc[2][kWarpsMax];         // per-warp counts, by round parity
  int wm[kWarpsMax];            // per-warp counts (compaction movers)
  int hist[3][kBins];
  int hsum[kBins];
  float smp_w[kWarpsMax];       // sampling: per-warp weight sums
  int smp_c, smp_pos;           // sampling: last kept candidate, drawn candidate
  float smp_ec;                 // sampling: weight sum of the kept candidates
  unsigned r_kmax, r_kmin;      // row-resident kernel: the row's largest and smallest keys,
  unsigned r_gmin;              //   the smallest vector maximum,
  unsigned r_tkey;              //   the k-th largest key and
  int r_ngt;                    //   how many keys exceed it
#ifdef DSEL_STATS
  unsigned long long st_compact_cycles;
  int st_compactions;
  int st_appended;
  int st_slow_vectors;
  int st_refetch;                 // passes restarted because a sampled seed was not certified
#endif
};

static_assert(offsetof(Ctl, hsum) % 16 == 0 && sizeof(Ctl::hsum) >= kTieMax * 8,
              "the radix select's small-bucket list fits hsum");
static_assert(offsetof(Ctl, hist) % 16 == 0 && (kBins * 4) % 16 == 0, "histograms are read as int4");

// Composite threshold word: larger means "ranks earlier".
__device__ __forceinline__ unsigned long long make_w(uint32_t key, uint32_t idx) {
  return (static_cast<unsigned long long>(key) << 32) | static_cast<uint32_t>(~idx);
}

// Radix word V = key << idx_bits | (idx_mask - idx): larger V ranks earlier and
// V is unique within a row.
__device__ __forceinline__ uint32_t mask_bits(int b) { return b >= 32 ? 0xFFFFFFFFu : ((1u << b) - 1u); }

template <int DT>
__device__ __forceinline__ uint64_t make_v(uint32_t bits, uint32_t idx, int idx_bits,
                                           uint32_t idx_mask) {
  return (static_cast<uint64_t>(Elem<DT>::key(bits)) << idx_bits) | (idx_mask - idx);
}

struct SelResult {
  uint64_t prefix;   // the kept candidates are those whose top `depth` bits of V are >= prefix
  int depth;
  int kept;          // how many they are (over the whole cluster in cluster mode)
};

// Warp-inclusive scan.
__device__ __forceinline__ int warp_incl_scan(int x, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  return x;
}

__device__ __forceinline__ uint64_t warp_max_u64(uint64_t v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const uint64_t y = __shfl_xor_sync(0xffffffffu, v, o);
    v = y > v ? y : v;
  }
  return v;
}

// Sum of per-warp values wc[0..NW) and the exclusive prefix for warp `warp`,
// computed by every warp on its own (no barrier).
template <int NW>
__device__ __forceinline__ int warp_prefix_of(const int* wc, int warp, int lane, int& total) {
  const int c = lane < NW ? wc[lane] : 0;
  const int incl = warp_incl_scan(c, lane);
  total = __shfl_sync(0xffffffffu, incl, 31);
  const int mine = __shfl_sync(0xffffffffu, incl - c, warp);
  return mine;
}

// Sum of lane `lane`'s contiguous chunk of N4 int4s, h4[base4 + lane * N4 ..
// + N4), read in a rotated order: with chunks of 2^m int4s the plain order puts
// up to 32 lanes on the same banks, the rotation keeps 8 lanes per wavefront
// (the minimum for 128-bit loads).  h4 must be 16-byte aligned.
template <int N4>
__device__ __forceinline__ int chunk_sum4(const int4* h4, int base4, int lane) {
  static_assert(N4 == 1 || N4 == 2 || N4 == 4 || N4 == 8, "chunk of 1, 2, 4 or 8 int4s");
  const int rot = (lane / (8 / N4)) % N4;
  int s = 0;
#pragma unroll
  for (int j = 0; j < N4; ++j) {
    const int4 q = h4[base4 + lane * N4 + ((j + rot) % N4)];
    s += q.x + q.y + q.z + q.w;
  }
  return s;
}

template <bool CLUSTER>
__device__ __forceinline__ void cta_or_cluster_sync(cg::cluster_group& cluster) {
  if (CLUSTER) cluster.sync();
  else __syncthreads();
}

// --------------------------------------------------------------------------- //
// MSB-first radix select over V.  Finds (prefix, depth) such that the candidates
// whose top `depth` bits are >= prefix number at least `need` and at most
// need + slack (exactly `need` with slack 0).  All candidates lie in [vlo, vhi],
// so the bits those two share are skipped.  One barrier per digit: histograms
// rotate over three buffers (build one, zero the next, the third may still be
// read), and every warp finds the bucket on its own.  While the digit lies in
// the key bits the arithmetic is 32-bit.  In cluster mode every CTA holds part
// of the candidates; histograms are summed over the cluster through distributed
// shared memory and every CTA takes the same decision.
// --------------------------------------------------------------------------- //
template <int DT, int THREADS, bool CLUSTER>
__device__ __noinline__ SelResult radix_select(const typename Elem<DT>::bits_t* cb, const uint32_t* ci, int cnt,
                                  const int need0, int slack, int idx_bits, uint64_t vlo, uint64_t vhi,
                                  Ctl& ctl, cg::cluster_group& cluster) {
  using E = Elem<DT>;
  const int tid = threadIdx.x, lane = tid & 31;
  const int total_bits = E::kKeyBits + idx_bits;
  const uint32_t idx_mask = mask_bits(idx_bits);
  int depth = vlo != vhi ? total_bits - (64 - __clzll(static_cast<long long>(vlo ^ vhi))) : total_bits;
  uint64_t prefix = depth == 0 ? 0ull : (vhi >> (total_bits - depth));
  if (depth >= total_bits) return {vhi, total_bits, need0};
  int need = need0;
  int hb = ctl.hb;
  int kept = need0;
  if (!CLUSTER && tid == 0) ctl.tie_n = 0;   // ordered before any use by the first pass's barrier
  while (true) {
    const int dbits = min(kDigitBits, total_bits - depth);
    const int shift = total_bits - depth - dbits;
    const uint32_t dmask = (1u << dbits) - 1u;
    int* h = ctl.hist[hb];
    int* hz = ctl.hist[hb == 2 ? 0 : hb + 1];
#pragma unroll 1
    for (int i = tid; i < kBins; i += THREADS) hz[i] = 0;
    if (shift >= idx_bits) {   // digit and prefix inside the key bits
      const int ks = shift - idx_bits;
      const uint32_t kp = static_cast<uint32_t>(prefix);
      const int ps = ks + dbits;   // < 32 here
#pragma unroll 4
      for (int i = tid; i < cnt; i += THREADS) {
        const uint32_t key = E::key(cb[i]);
        if ((ps >= 32 ? 0u : (key >> ps)) == kp) atomicAdd(&h[(key >> ks) & dmask], 1);
      }
    } else {
#pragma unroll 4
      for (int i = tid; i < cnt; i += THREADS) {
        const uint64_t v = make_v<DT>(cb[i], ci[i], idx_bits, idx_mask);
        if ((v >> (shift + dbits)) == prefix) atomicAdd(&h[static_cast<uint32_t>(v >> shift) & dmask], 1);
      }
    }
    const int* H = h;
    cta_or_cluster_sync<CLUSTER>(cluster);
    if (CLUSTER) {
      const int nr = static_cast<int>(cluster.num_blocks());
#pragma unroll 1
      for (int b = tid; b < kBins; b += THREADS) {
        int s = 0;
#pragma unroll 1
        for (int r = 0; r < nr; ++r) s += cluster.map_shared_rank(h, r)[b];
        ctl.hsum[b] = s;
      }
      __syncthreads();
      H = ctl.hsum;
    }
    // every warp: bins from the top, 8 per lane, find the bucket holding the need-th
    // lane l holds bins kBins-1-8l down to kBins-8-8l (c[0] the highest), read as
    // two int4s whose order alternates between lane groups (no bank conflicts)
    static_assert(kBins == 256, "two int4s of bins per lane");
    int c[8];
    {
      const int4* H4 = reinterpret_cast<const int4*>(H);
      const int sw = (lane >> 2) & 1;
      const int4 qa = H4[62 - 2 * lane + sw];
      const int4 qb = H4[63 - 2 * lane - sw];
      const int4 lo = sw ? qb : qa, hi = sw ? qa : qb;   // bins 248-8l.. and 252-8l..
      c[0] = hi.w; c[1] = hi.z; c[2] = hi.y; c[3] = hi.x;
      c[4] = lo.w; c[5] = lo.z; c[6] = lo.y; c[7] = lo.x;
    }
    int s = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) s += c[j];
    const int incl = warp_incl_scan(s, lane);
    const int excl = incl - s;
    const bool mine = excl < need && need <= incl;
    int digit = 0, above = 0, bucket = 0;
    if (mine) {
      int acc = excl;
      bool done = false;
#pragma unroll
      for (int j = 0; j < kBins / 32; ++j) {
        if (!done && acc + c[j] >= need) {
          digit = kBins - 1 - (lane * (kBins / 32) + j);
          above = acc;
          bucket = c[j];
          done = true;
        }
        acc += c[j];
      }
    }
    const int src = __ffs(__ballot_sync(0xffffffffu, mine)) - 1;
    digit = __shfl_sync(0xffffffffu, digit, src);
    above = __shfl_sync(0xffffffffu, above, src);
    bucket = __shfl_sync(0xffffffffu, bucket, src);
    need -= above;
    prefix = (prefix << dbits) | static_cast<uint64_t>(digit);
    depth += dbits;
    hb = hb == 2 ? 0 : hb + 1;
    kept = need0 - need + bucket;
    if (bucket - need <= slack || depth == total_bits) break;
    if (!CLUSTER && slack == 0 && bucket <= kTieMax) {
      // Small bucket (typically equal keys at the boundary): rank its members by
      // their whole radix word, which is unique, instead of more digit passes.
      unsigned long long* lst = reinterpret_cast<unsigned long long*>(ctl.hsum);
      const int sh = total_bits - depth;
#pragma unroll 1
      for (int i0 = 0; i0 < cnt; i0 += THREADS) {   // same trip count in every thread
        const int i = i0 + tid;
        uint64_t v = 0;
        bool in = false;
        if (i < cnt) {
          v = make_v<DT>(cb[i], ci[i], idx_bits, idx_mask);
          in = (v >> sh) == prefix;
        }
        const unsigned bal = __ballot_sync(0xffffffffu, in);
        int base = 0;
        if (lane == 0 && bal != 0u) base = atomicAdd(&ctl.tie_n, __popc(bal));
        base = __shfl_sync(0xffffffffu, base, 0);
        if (in) lst[base + __popc(bal & ((1u << lane) - 1u))] = v;
      }
      __syncthreads();
      if (tid < bucket) {   // the member with need - 1 larger words is the need-th
        const unsigned long long vj = lst[tid];
        int r = 0;
#pragma unroll 4
        for (int i = 0; i < bucket; ++i) r += lst[i] > vj ? 1 : 0;
        if (r == need - 1) ctl.tie_v = vj;
      }
      __syncthreads();
      prefix = ctl.tie_v;
      depth = total_bits;
      kept = need0;
      break;
    }
  }
  if (tid == 0) ctl.hb = hb;   // read again only after later barriers
  return {prefix, depth, kept};
}

// The need-th largest radix word among the n candidates whose key lies in
// [klo, khi] (at most kTieMax of them, `members`): gathered into a short list,
// each ranked by its whole word, which is unique.  ctl.tie_n must be zero on
// entry and ordered by an earlier barrier.  Two barriers.
template <int DT, int THREADS>
__device__ __noinline__ uint64_t rank_members(const typename Elem<DT>::bits_t* cb, const uint32_t* ci, int n,
                                              uint32_t klo, uint32_t khi, int members, int need, int idx_bits,
                                              Ctl& ctl) {
  const int tid = threadIdx.x, lane = tid & 31;
  const uint32_t idx_mask = mask_bits(idx_bits);
  unsigned long long* lst = reinterpret_cast<unsigned long long*>(ctl.hsum);
#pragma unroll 1
  for (int i0 = 0; i0 < n; i0 += THREADS) {   // same trip count in every thread
    const int i = i0 + tid;
    uint64_t v = 0;
    bool in = false;
    if (i < n) {
      const uint32_t key = Elem<DT>::key(cb[i]);
      in = key >= klo && key <= khi;
      v = make_v<DT>(cb[i], ci[i], idx_bits, idx_mask);
    }
    const unsigned bal = __ballot_sync(0xffffffffu, in);
    int base = 0;
    if (lane == 0 && bal != 0u) base = atomicAdd(&ctl.tie_n, __popc(bal));
    base = __shfl_sync(0xffffffffu, base, 0);
    if (in) lst[base + __popc(bal & ((1u << lane) - 1u))] = v;
  }
  __syncthreads();
  if (tid < members) {   // the member with need - 1 larger words is the need-th
    const unsigned long long vj = lst[tid];
    int r = 0;
#pragma unroll 4
    for (int i = 0; i < members; ++i) r += lst[i] > vj ? 1 : 0;
    if (r == need - 1) ctl.tie_v = vj;
  }
  __syncthreads();
  return ctl.tie_v;
}

// Exact selection of the k best of n candidates (all radix words in [vlo, vhi]),
// as a SelResult, starting with one pass of a histogram of 1024 bins spread
// evenly over the candidates' key range (bins of 2^sh keys; one key per bin when
// the range is under 1024 keys, as bf16 candidates usually are).  Radix digits
// aligned to key bits put the first digit on the exponent, so on data with few
// distinct values nearly all candidates fall into one or two bins and their
// atomics serialise; the range-adaptive bins do not.  The boundary bin is then
// finished by ranking its members (at most kTieMax) or, failing that, by the
// radix select (restricted to the boundary key when bins are single keys).
// `hist` is 1024 ints of scratch, 16-byte aligned.
template <int DT, int THREADS>
__device__ __noinline__ SelResult select_by_key_hist(const typename Elem<DT>::bits_t* cb, const uint32_t* ci, int n,
                                                     int k, int idx_bits, uint64_t vlo, uint64_t vhi, Ctl& ctl,
                                                     int* hist, cg::cluster_group& cluster) {
  using E = Elem<DT>;
  constexpr int NB = 1024;
  const int tid = threadIdx.x, lane = tid & 31;
  const int total_bits = E::kKeyBits + idx_bits;
  const uint32_t kmin = static_cast<uint32_t>(vlo >> idx_bits), kmax = static_cast<uint32_t>(vhi >> idx_bits);
  const int sh = max(0, (32 - __clz(kmax - kmin)) - 10);   // ((kmax - kmin) >> sh) < NB
#pragma unroll 1
  for (int i = tid; i < NB; i += THREADS) hist[i] = 0;
  if (tid == 0) ctl.tie_n = 0;
  __syncthreads();
#pragma unroll 1
  for (int i = tid; i < n; i += THREADS)   // the clamp only guards the array: keys lie in [kmin, kmax]
    atomicAdd(&hist[min((E::key(cb[i]) - kmin) >> sh, static_cast<uint32_t>(NB - 1))], 1);
  __syncthreads();
  // every warp: lane l sums bins NB-32-32l .. NB-1-32l (int4s 8(31-l) ..), scans,
  // and the lane holding the k-th largest walks its bins from the top
  const int top = NB - 1 - lane * 32;
  const int sum = chunk_sum4<8>(reinterpret_cast<const int4*>(hist), 0, 31 - lane);
  const int incl = warp_incl_scan(sum, lane);
  const bool mine = incl - sum < k && k <= incl;
  int bin = 0, above = 0;
  if (mine) {
    int acc = incl - sum;
#pragma unroll 1
    for (int j = 0; j < 32; ++j) {
      const int c = hist[top - j];
      if (acc + c >= k) {
        bin = top - j;
        above = acc;
        break;
      }
      acc += c;
    }
  }
  const int src = __ffs(__ballot_sync(0xffffffffu, mine)) - 1;
  bin = __shfl_sync(0xffffffffu, bin, src);
  above = __shfl_sync(0xffffffffu, above, src);
  const int bucket = hist[bin];
  const int need = k - above;
  const uint32_t klo = kmin + (static_cast<uint32_t>(bin) << sh);
  if (sh == 0) {   // the boundary bin is one key
    if (bucket == need) return SelResult{klo, E::kKeyBits, k};   // every candidate of that key is kept
    if (bucket <= kTieMax)
      return SelResult{rank_members<DT, THREADS>(cb, ci, n, klo, klo, bucket, need, idx_bits, ctl), total_bits, k};
    // many candidates of that key: their index digits
    const uint32_t idx_mask = mask_bits(idx_bits);
    const uint64_t base = static_cast<uint64_t>(klo) << idx_bits;
    const SelResult r =
        radix_select<DT, THREADS, false>(cb, ci, n, need, 0, idx_bits, base, base | idx_mask, ctl, cluster);
    return SelResult{r.prefix, r.depth, k};
  }
  if (bucket <= kTieMax) {
    const uint32_t khi = klo + ((1u << sh) - 1u);
    return SelResult{rank_members<DT, THREADS>(cb, ci, n, klo, khi, bucket, need, idx_bits, ctl), total_bits, k};
  }
  return radix_select<DT, THREADS, false>(cb, ci, n, k, 0, idx_bits, vlo, vhi, ctl, cluster);
}

// Keep the candidates whose top `depth` bits are >= prefix (`kept` of them, or
// counted here when kept < 0), moving those found past position kept into the
// holes below it.  Order is not preserved; positions come from per-warp counts
// (no atomics), each warp owning a contiguous chunk.  Returns the kept count.
template <int DT, int THREADS>
__device__ __noinline__ int holes_compact(typename Elem<DT>::bits_t* cb, uint32_t* ci, int cnt, int kept,
                             SelResult sel, int idx_bits, Ctl& ctl, uint32_t* holes) {
  constexpr int NW = THREADS / 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int sh = Elem<DT>::kKeyBits + idx_bits - sel.depth;
  const uint32_t idx_mask = mask_bits(idx_bits);
  auto keep_at = [&](int p) -> bool {
    return (make_v<DT>(cb[p], ci[p], idx_bits, idx_mask) >> sh) >= sel.prefix;
  };
  if (kept < 0) {   // count first
    const int chunk = ((cnt + NW - 1) / NW + 31) & ~31;
    const int a = min(cnt, warp * chunk), b = min(cnt, a + chunk);
    int n = 0;
#pragma unroll 1
    for (int p0 = a; p0 < b; p0 += 32) {
      const int p = p0 + lane;
      n += __popc(__ballot_sync(0xffffffffu, p < b && keep_at(p)));
    }
    if (lane == 0) ctl.wm[warp] = n;
    __syncthreads();
    int total;
    warp_prefix_of<NW>(ctl.wm, warp, lane, total);
    kept = total;
    __syncthreads();
  }
  // holes live in [0, kept), movers in [kept, cnt)
  const int hc = ((kept + NW - 1) / NW + 31) & ~31;
  const int mc = ((cnt - kept + NW - 1) / NW + 31) & ~31;
  const int ha = min(kept, warp * hc), hbnd = min(kept, ha + hc);
  const int ma = kept + min(cnt - kept, warp * mc), mbnd = min(cnt, ma + mc);
  int nh = 0, nm = 0;
#pragma unroll 1
  for (int p0 = ha; p0 < hbnd; p0 += 32) {
    const int p = p0 + lane;
    nh += __popc(__ballot_sync(0xffffffffu, p < hbnd && !keep_at(p)));
  }
#pragma unroll 1
  for (int p0 = ma; p0 < mbnd; p0 += 32) {
    const int p = p0 + lane;
    nm += __popc(__ballot_sync(0xffffffffu, p < mbnd && keep_at(p)));
  }
  if (lane == 0) {
    ctl.wc[0][warp] = nh;
    ctl.wm[warp] = nm;
  }
  __syncthreads();
  int tot;
  int hoff = warp_prefix_of<NW>(ctl.wc[0], warp, lane, tot);
  int moff = warp_prefix_of<NW>(ctl.wm, warp, lane, tot);
  const uint32_t below = (1u << lane) - 1u;
#pragma unroll 1
  for (int p0 = ha; p0 < hbnd; p0 += 32) {
    const int p = p0 + lane;
    const bool hole = p < hbnd && !keep_at(p);
    const uint32_t bal = __ballot_sync(0xffffffffu, hole);
    if (hole) holes[hoff + __popc(bal & below)] = static_cast<uint32_t>(p);
    hoff += __popc(bal);
  }
  __syncthreads();
#pragma unroll 1
  for (int p0 = ma; p0 < mbnd; p0 += 32) {
    const int p = p0 + lane;
    const bool mover = p < mbnd && keep_at(p);
    const uint32_t bal = __ballot_sync(0xffffffffu, mover);
    if (mover) {
      const uint32_t q = holes[moff + __popc(bal & below)];
      cb[q] = cb[p];
      ci[q] = ci[p];
    }
    moff += __popc(bal);
  }
  __syncthreads();
  return kept;
}

// Threshold word for a selection result: the smallest V with that prefix.
__device__ __forceinline__ uint64_t v_floor(SelResult sel, int total_bits) {
  return sel.prefix << (total_bits - sel.depth);
}

__device__ __forceinline__ unsigned long long threshold_of(SelResult sel, int key_bits, int idx_bits) {
  const uint32_t idx_mask = mask_bits(idx_bits);
  const uint64_t v = v_floor(sel, key_bits + idx_bits);
  const uint32_t key = static_cast<uint32_t>(v >> idx_bits);
  const uint32_t rev = static_cast<uint32_t>(v) & idx_mask;
  return make_w(key, idx_mask - rev);
}

// Bitonic sort of m (<= capacity, padded to a power of two) candidates in shared
// memory.  BY_VALUE: value descending, then index ascending; else index ascending.
template <int DT, int THREADS, bool BY_VALUE>
__device__ __noinline__ void bitonic_sort(typename Elem<DT>::bits_t* cb, uint32_t* ci, int m) {
  const int tid = threadIdx.x;
  int M = 1;
  while (M < m) M <<= 1;
  // padding: index 0xFFFFFFFF and the all-ones pattern (key 0, below every real key,
  // a negative NaN included), so it sorts after every real entry in either order
#pragma unroll 1
  for (int i = m + tid; i < M; i += THREADS) {
    ci[i] = 0xFFFFFFFFu;
    cb[i] = static_cast<typename Elem<DT>::bits_t>(~0u);
  }
  __syncthreads();
#pragma unroll 1
  for (int size = 2; size <= M; size <<= 1) {
#pragma unroll 1
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
#pragma unroll 1
      for (int t = tid; t < (M >> 1); t += THREADS) {
        const int lo = 2 * t - (t & (stride - 1));
        const int hi = lo + stride;
        const bool asc = (lo & size) == 0;
        const uint32_t ia = ci[lo], ib = ci[hi];
        bool gt;
        if (BY_VALUE) {
          // sort key ascending = (inverted key, index): value desc then index asc.
          // Padding (index 0xFFFFFFFF, -inf) lands after every real entry.
          const uint64_t ka = (static_cast<uint64_t>(~Elem<DT>::key(cb[lo])) << 32) | ia;
          const uint64_t kb = (static_cast<uint64_t>(~Elem<DT>::key(cb[hi])) << 32) | ib;
          gt = ka > kb;
        } else {
          gt = ia > ib;
        }
        if (gt == asc) {
          const auto ba = cb[lo];
          cb[lo] = cb[hi];
          cb[hi] = ba;
          ci[lo] = ib;
          ci[hi] = ia;
        }
      }
      __syncthreads();
    }
  }
}

}  // namespace dsel
