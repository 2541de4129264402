// Host-side launch planner for the row-wise TopK kernels.  Pure C++: no CUDA call,
// so it is unit-tested on machines without a GPU through dsel_plan().
#pragma once
#include <algorithm>
#include <cstdint>

#include "../../include/dsel.h"

namespace dsel {

// Compile-time CTA shapes.  The streaming kernel is instantiated for exactly
// these (dtype, threads) pairs; the planner only ever returns one of them:
// 512 threads, one CTA per SM, for long rows and split rows; 256 threads, two per
// SM, for batches of long rows with k <= 1024; 128 threads for many short rows,
// so that several rows share an SM and one CTA's loads overlap another's work.
constexpr int kThreads = 512;
constexpr int kThreadsMid = 256;
constexpr int kThreadsShort = 128;
constexpr int kVecBytes = 16;                 // one 128-bit shared-memory load per vector
// Row-resident kernel: one 256-thread CTA per row holds the whole row (at most
// 32 KB: 16,384 bf16 or 8,192 f32 elements) in shared memory.
constexpr int kResThreads = 256;
constexpr int kResRowBytes = 32 * 1024;
// Slice-resident kernel: one CTA per slice of a row (at most 8 chunks of 16 KB:
// 128 KB), the slices of a row in one thread-block cluster.  512 threads (two
// 16-byte vectors per thread and chunk) for slices of four chunks or more, whose
// per-vector passes need the warps to hide their latency; 256 threads (four
// vectors per thread and chunk) for smaller slices, where the fixed per-CTA work
// dominates.
constexpr int kSliceThreadsLarge = 512;
constexpr int kSliceThreadsSmall = 256;
constexpr int kSliceLargeFromChunks = 4;
constexpr int slice_threads(int64_t chunks) {
  return chunks >= kSliceLargeFromChunks ? kSliceThreadsLarge : kSliceThreadsSmall;
}
constexpr int kSliceChunkBytes = 16384;
constexpr int kSliceMaxChunks = 8;
constexpr int kSliceMaxCluster = 16;          // non-portable cluster size (B200 schedules 16)
constexpr int kSliceMinElems = 8192;          // smallest slice worth its own CTA
constexpr int kSliceMaxWaves = 4;             // batches of more slices than this many SM waves stream
constexpr int kSliceCtlBytes = 1024;          // its control block
constexpr int kSliceMaxList = 16384;          // candidate-list entries
// list entries beyond k a slice plan must hold: room for keys equal to the
// threshold when one slice holds a sorted row's whole top k (2000 rather than
// 2048 lets 64 rows of 129,280 f32 at k = 4096 take clusters of 4, two waves of
// slices instead of three)
constexpr int kSliceListSlack = 2000;
// Vectors each thread screens per round (a warp owns whole blocks): 16 for bf16
// (a 64K-element round, the whole slice of a 131,072-position row split in two),
// 8 for f32 (16K elements, so that two rounds fit the ring for double buffering).
constexpr int vecs_per_thread_for(int eb) { return eb == 2 ? 16 : 8; }

// Candidate-buffer slots beyond k + B2.  A round's survivors that do not fit
// wait until a compaction makes room, so this need not cover a whole round.
inline int append_slack(int k, int threads) {
  if (threads != kThreads) return 1024;
  return k <= 1024 ? 4096 : 2048;
}
constexpr int kSeedSlots = 4096;              // candidate slots that hold the round-0 seed histograms
constexpr int kStrideReq = 16;                // row_stride multiple (elements)
constexpr int kMaxStages = 128;               // ring depth cap (one mbarrier per stage)
constexpr int kMinSliceElems = 8192;          // smallest row share worth its own CTA
constexpr int kSharedFixedBytes = 6144;       // control block: scalars, histograms, scan scratch
constexpr int kMaxK = 4096;
constexpr int kMaxCluster = 8;                // portable cluster size
constexpr int kMaxGroups = 255;               // clusters per row (merge keeps one prefix per group)

inline int elem_bytes(int dtype) { return dtype == DSEL_BF16 ? 2 : 4; }

// Elements a CTA filters between two checks of the candidate buffer.
constexpr int round_elems_for(int eb, int threads) { return threads * vecs_per_thread_for(eb) * (kVecBytes / eb); }
inline int round_elems(int dtype, int threads) { return round_elems_for(elem_bytes(dtype), threads); }

// B, elements per contiguous block (the unit of the random visiting order and of
// one bulk copy): one warp's share of a round, 32 lanes x vectors per thread, so
// each warp issues, and waits on, exactly one copy per round.  4096 for bf16
// (8 KB), 1024 for f32 (4 KB).  The pages set B = 1024 for k = 512; bf16 takes
// the larger block so that a CTA issues a quarter as many copies.
constexpr int block_elems_for(int eb) { return 32 * vecs_per_thread_for(eb) * (kVecBytes / eb); }
inline int block_elems(int dtype) { return block_elems_for(elem_bytes(dtype)); }

inline int ceil_log2_u64(uint64_t v) {   // smallest b with 2^b >= v (v >= 1)
  int b = 0;
  while ((uint64_t(1) << b) < v) ++b;
  return b;
}

inline int next_pow2(int v) {
  int p = 1;
  while (p < v) p <<= 1;
  return p;
}

// CTAs per row in the merge launch of a split-row plan: enough that each holds at
// most `capacity` of the groups' partial results.
inline int merge_cluster(const dsel_plan_t& p, int k) {
  const int64_t total = int64_t(p.groups) * k;
  int c = int((total + p.capacity - 1) / p.capacity);
  if (c < 1) c = 1;
  if (c > kMaxCluster) c = kMaxCluster;
  return c;
}

// Shared-memory layout of the kernels (byte offsets from the dynamic
// shared-memory base).  The device code receives these offsets; nothing on the
// device recomputes them.
struct SmemLayout {
  uint32_t bars, blk, cb, ci, holes, ctl, total;
};

// `holes` = slots of the compaction hole list (k + B2: a compaction keeps at most k + B2/2).
inline SmemLayout stream_layout(int64_t stages, int64_t block, int64_t capacity, int64_t holes, int eb) {
  auto up = [](int64_t v, int64_t a) { return (v + a - 1) / a * a; };
  SmemLayout l{};
  int64_t off = up(stages * block * eb, 128);
  l.bars = uint32_t(off);
  off += up(stages * 8, 16);
  l.blk = uint32_t(off);
  off += up(stages * 4, 16);
  l.cb = uint32_t(off);
  off += up(capacity * eb, 16);
  l.ci = uint32_t(off);
  off += up(capacity * 4, 16);
  l.holes = uint32_t(off);
  off += up(holes * 4, 16);
  l.ctl = uint32_t(off);
  off += kSharedFixedBytes;
  l.total = uint32_t(off);
  return l;
}

// Row-resident kernel: the row; one mbarrier per 4 KB chunk (256 threads x 16
// bytes); two 1024-bin histograms followed by the per-warp candidate lists (16-bit
// row indices, at least 4 KB: the exact fallback keeps a third histogram there);
// the row's candidate vectors (16-bit vector indices; the fallback's 512-byte
// scan table in the same space); candidate arrays of next_pow2(k) entries (value
// order and the sampling step sort there); the control block.  The lists take
// what shared memory is left below the size that keeps the most CTAs on an SM (at
// most four: 256 threads of at most 64 registers), and no more than a warp can
// fill (its share of the row's vectors, every element a candidate).
constexpr int kResCtlBytes = 1024;
constexpr int kResMaxCtasPerSm = 4;
constexpr int kResMinListBytes = 4096;
constexpr int64_t kSmemPerSm = 228 * 1024;        // B200: shared memory per SM
constexpr int64_t kSmemReservedPerCta = 1024;     // reserved by the system for every resident CTA

struct ResLayout {
  uint32_t bars, hist, el, vl, cb, ci, ctl, total;
  int32_t seg;   // list entries per warp
};

inline ResLayout resident_layout(int64_t row_stride, int32_t k, int eb) {
  auto up = [](int64_t v, int64_t a) { return (v + a - 1) / a * a; };
  const int vpt = kResRowBytes / (kResThreads * kVecBytes);
  const int nw = kResThreads / 32;
  const int pv = kVecBytes / eb;
  const int64_t nvec = (row_stride + pv - 1) / pv;
  const int64_t kp2 = next_pow2(k);
  const int64_t row = up(row_stride * eb, 128);
  const int64_t bars = up(int64_t(vpt) * 8, 16);
  const int64_t hist = 2 * 1024 * 4;
  const int64_t vl = std::max<int64_t>(up(nvec * 2, 16), 2 * int64_t(vpt) * nw * 4);
  const int64_t cbb = up(kp2 * eb, 16), cib = up(kp2 * 4, 16);
  const int64_t fixed = row + bars + hist + vl + cbb + cib + kResCtlBytes;
  int occ = kResMaxCtasPerSm;
  while (occ > 1 && occ * (fixed + kResMinListBytes + kSmemReservedPerCta) > kSmemPerSm) --occ;
  const int64_t budget = kSmemPerSm / occ - kSmemReservedPerCta - fixed;
  const int64_t full = 2 * nw * ((nvec + nw - 1) / nw) * pv;   // every element of a warp's share
  int64_t el = std::min<int64_t>(std::max<int64_t>(budget, kResMinListBytes), std::max<int64_t>(full, kResMinListBytes));
  const int64_t seg = el / (2 * nw);
  el = up(seg * 2 * nw, 16);
  ResLayout l{};
  int64_t off = row;
  l.bars = uint32_t(off);
  off += bars;
  l.hist = uint32_t(off);
  off += hist;
  l.el = uint32_t(off);   // right after the histograms: the fallback's third buffer
  off += el;
  l.vl = uint32_t(off);
  off += vl;
  l.cb = uint32_t(off);
  off += cbb;
  l.ci = uint32_t(off);
  off += cib;
  l.ctl = uint32_t(off);
  off += kResCtlBytes;
  l.total = uint32_t(off);
  l.seg = int32_t(seg);
  return l;
}

// Slice kernel: the slice (chunks of 16 KB), the 16-bit maxima of its vectors
// (later the bitmap ranks: 2 KB per chunk either way), one mbarrier per chunk, the
// CTA's candidate lists (elements: bits and row index; vectors: half as many
// indices), a 4096-bin histogram of the vector maxima and a 1024-bin one of the
// candidates, and the control block.
struct SliceLayout {
  uint32_t tab, bars, cb, ci, cv, hist, ctl, total;
};

inline SliceLayout slice_layout(int64_t chunks, int64_t lcap, int eb) {
  auto up = [](int64_t v, int64_t a) { return (v + a - 1) / a * a; };
  SliceLayout l{};
  int64_t off = chunks * kSliceChunkBytes;
  l.tab = uint32_t(off);
  off += chunks * (kSliceChunkBytes / kVecBytes) * 2;   // a 16-bit summary per vector
  l.bars = uint32_t(off);
  off += up(chunks * 8, 16);
  l.cb = uint32_t(off);
  off += up(lcap * eb, 16);
  l.ci = uint32_t(off);
  off += up(lcap * 4, 16);
  l.cv = uint32_t(off);   // candidate vectors: half as many entries as the element list
  off += up(lcap / 2 * 4, 16);
  l.hist = uint32_t(off);
  off += (4096 + 1024 + 512) * 4;   // and their coarse sums
  l.ctl = uint32_t(off);
  off += kSliceCtlBytes;
  l.total = uint32_t(off);
  return l;
}

#ifdef __CUDACC__
#define DSEL_HOST_DEVICE __host__ __device__
#else
#define DSEL_HOST_DEVICE
#endif

// Visiting stride of n chunks: about 0.618 n, odd, coprime with n (1 for n <= 2).
// Host and device: the host computes it for rows of row_stride elements, a
// kernel for a row that `end` shortens.
DSEL_HOST_DEVICE inline uint32_t chunk_stride(uint32_t n) {
  if (n <= 2) return 1u;
  uint32_t a = (n * 618u + 500u) / 1000u | 1u;
  for (;; a += 2u) {
    uint32_t x = a, y = n;
    while (y) {
      const uint32_t t = x % y;
      x = y;
      y = t;
    }
    if (x == 1u) break;
  }
  return a % n;
}

// Chunks of a slice of ceil(row_stride / C) elements (rounded up to 16).
inline int64_t slice_chunks(int64_t row_stride, int64_t C, int eb) {
  const int64_t sl = ((row_stride + C - 1) / C + 15) / 16 * 16;
  const int64_t per = kSliceChunkBytes / eb;
  return (sl + per - 1) / per;
}

// Candidate-list entries that fit next to `chunks` chunks in `smem` bytes.
inline int64_t slice_list_cap(int64_t chunks, int64_t smem, int eb) {
  const int64_t fixed = slice_layout(chunks, 0, eb).total + 64;
  int64_t l = (smem - fixed) / (eb + 4 + 2);
  l = l < kSliceMaxList ? l : kSliceMaxList;
  return l / 32 * 32;
}

// Merge kernel: candidate arrays, hole list and the control block.
inline SmemLayout merge_layout(int64_t capacity, int64_t holes, int eb) {
  auto up = [](int64_t v, int64_t a) { return (v + a - 1) / a * a; };
  SmemLayout l{};
  int64_t off = 0;
  l.cb = 0;
  off += up(capacity * eb, 16);
  l.ci = uint32_t(off);
  off += up(capacity * 4, 16);
  l.holes = uint32_t(off);
  off += up(holes * 4, 16);
  l.ctl = uint32_t(off);
  off += kSharedFixedBytes;
  l.total = uint32_t(off);
  return l;
}

int make_plan(int dtype, int64_t rows, int64_t row_stride, int32_t k, int32_t num_sms,
              int32_t smem_optin, int32_t max_cluster, dsel_plan_t* out);

// make_plan with control over the slice kernel: `slice_cluster` is the largest
// cluster the slice kernel may use (0: never use it, as for value order and the
// sampling step, which the other kernels serve).  `cluster_fit`, when given, holds
// for each cluster size c in [1, kSliceMaxCluster] how many clusters of c streaming
// CTAs the device holds at once: a split row then takes the cluster size and
// number of groups with the most CTAs whose clusters all fit at once (one wave).
int make_plan_ex(int dtype, int64_t rows, int64_t row_stride, int32_t k, int32_t num_sms,
                 int32_t smem_optin, int32_t max_cluster, int32_t slice_cluster, dsel_plan_t* out,
                 const int32_t* cluster_fit = nullptr);

// Argument checks shared by dsel_topk and dsel_plan (host only).
int check_shape(int dtype, int64_t rows, int64_t row_stride, int32_t k);

}  // namespace dsel
