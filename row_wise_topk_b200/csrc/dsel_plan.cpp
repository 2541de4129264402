// Launch planner: picks the CTA shape, the row split and the ring depth.
//
// The pages fix only B = B2 = 1024 for k = 512 ("DeepSeek releases DeepSelect, a
// TopK kernel for sparse attention and sampling", method paragraph) and say both
// should sit "on the order of k"; B2 follows them, B is one warp's share of a
// round (4096 bf16 / 1024 f32 elements, see block_elems_for), and everything
// else here is this library's choice for a 148-SM B200:
//   * one CTA per row while there are at least as many rows as SMs:
//       - rows of at most 32 KB: the row-resident kernel (dsel_resident.cuh),
//         which holds the whole row in shared memory;
//       - rows of at most two 128-thread rounds: a 128-thread CTA, several per
//         SM, each with at most one round of blocks in flight;
//       - longer rows with k <= 1024: a 256-thread CTA when two fit an SM (two
//         rows per SM: one wave for up to 2 x SMs rows, and one CTA's barrier
//         waits overlap the other's work);
//       - otherwise a 512-thread CTA, one per SM;
//   * otherwise each row is cut into S contiguous slices, one CTA each, grouped in
//     thread-block clusters of C CTAs that share the threshold and merge through
//     distributed shared memory; rows too long for one cluster (S > max_cluster)
//     get G clusters and a second, merging launch;
//   * the shared-memory ring holds as many blocks in flight as fit next to the
//     candidate buffer (up to the whole slice).
#include "dsel_plan.h"

#include <algorithm>

namespace dsel {

int check_shape(int dtype, int64_t rows, int64_t row_stride, int32_t k) {
  if (dtype != DSEL_BF16 && dtype != DSEL_F32) return DSEL_ERR_DTYPE;
  if (k < 1 || k > kMaxK) return DSEL_ERR_K;
  if (rows < 0) return DSEL_ERR_ROWS;
  if (row_stride < 1 || row_stride > INT32_MAX || row_stride % kStrideReq != 0)
    return DSEL_ERR_STRIDE;
  return DSEL_OK;
}

static int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
static int64_t round_up(int64_t a, int64_t b) { return ceil_div(a, b) * b; }

namespace {

// Buffer sizes and block geometry for one CTA shape (ring depth still open).
void shape_plan(int dtype, int32_t k, int threads, dsel_plan_t* p) {
  p->threads = threads;
  p->block = block_elems(dtype);
  p->round = round_elems(dtype, threads);
  p->b2 = k <= 1024 ? 1024 : std::min(k, 2048);
  // k + B2 + slack; a round's survivors beyond that wait in registers until a
  // compaction makes room, so the round may be larger than the slack;
  // at least kSeedSlots: the round-0 seed histograms live in the index array
  p->capacity = int(round_up(
      std::max<int64_t>({int64_t(k) + p->b2 + append_slack(k, threads), int64_t(next_pow2(k)), int64_t(kSeedSlots)}),
      32));
}

int64_t shape_smem(const dsel_plan_t& p, int64_t stages, int32_t k, int eb) {
  return stream_layout(stages, p.block, p.capacity, int64_t(k) + p.b2, eb).total;
}

}  // namespace

int make_plan(int dtype, int64_t rows, int64_t row_stride, int32_t k, int32_t num_sms,
              int32_t smem_optin, int32_t max_cluster, dsel_plan_t* out) {
  return make_plan_ex(dtype, rows, row_stride, k, num_sms, smem_optin, max_cluster, kSliceMaxCluster, out);
}

int make_plan_ex(int dtype, int64_t rows, int64_t row_stride, int32_t k, int32_t num_sms,
                 int32_t smem_optin, int32_t max_cluster, int32_t slice_cluster, dsel_plan_t* out,
                 const int32_t* cluster_fit) {
  int st = check_shape(dtype, rows, row_stride, k);
  if (st != DSEL_OK) return st;
  if (out == nullptr || num_sms < 1 || smem_optin < 48 * 1024 || max_cluster < 1)
    return DSEL_ERR_DEVICE;

  const int eb = elem_bytes(dtype);
  dsel_plan_t p{};
  const bool one_per_row = rows >= num_sms;
  const bool resident_rows = one_per_row && row_stride * eb <= kResRowBytes;

  // Rows that fit in shared memory: the row-resident kernel.
  if (one_per_row && row_stride * eb <= kResRowBytes) {
    const ResLayout rl = resident_layout(row_stride, k, eb);
    if (int64_t(rl.total) <= smem_optin) {
      p.kernel = DSEL_KERNEL_RESIDENT;
      p.threads = kResThreads;
      p.cluster = 1;
      p.groups = 1;
      p.block = kResThreads * kVecBytes / eb;
      p.b2 = 0;
      p.round = int(row_stride);
      p.capacity = next_pow2(k);
      p.stages = int(ceil_div(row_stride * eb, int64_t(kResThreads) * kVecBytes));
      p.idx_bits = ceil_log2_u64(uint64_t(row_stride));
      p.smem_bytes = int(rl.total);
      p.workspace_bytes = 0;
      *out = p;
      return DSEL_OK;
    }
  }
  // Rows that fit, a few slices each, in the shared memory of one cluster: the
  // slice kernel.  The fewest slices that fit, or more while the batch leaves SMs
  // idle (but no slice under kSliceMinElems); the candidate list takes the rest of
  // the shared memory and must hold at least k + kSliceListSlack entries: a slice that holds
  // the whole top k (a sorted row) still fits its list, with room for the keys
  // equal to the threshold; a list that overflows sends the row to the exact
  // selection on the resident slices.
  if (slice_cluster >= 1 && !resident_rows) {
    auto fits = [&](int64_t c) {
      const int64_t ch = slice_chunks(row_stride, c, eb);
      return ch <= kSliceMaxChunks && slice_list_cap(ch, smem_optin, eb) >= int64_t(k) + kSliceListSlack;
    };
    int64_t cmin = 0;
    for (int64_t c = 1; c <= slice_cluster; ++c) {
      if (fits(c)) {
        cmin = c;
        break;
      }
    }
    // a few waves at most: a CTA holds its SM from the first copy to the last
    // write, so batches needing many waves of slices go to the streaming kernel,
    // whose two CTAs per SM overlap one row's tail with the next row's loads
    if (cmin > 0 && rows * cmin <= kSliceMaxWaves * int64_t(num_sms)) {
      // more slices than needed only to put idle SMs to work, and then at most the
      // portable 8: a cluster of 16 ranks has the longer finish (one row of 129,280
      // f32 logits: 10.3 us in 16 slices of 32 KB, 9.1 us in 8 of 64 KB; eight rows:
      // 25.2 against 12.7 us); rows that need more than 8 slices to fit keep cmin
      int64_t c = std::max<int64_t>(1, num_sms / std::max<int64_t>(rows, 1));
      c = std::min<int64_t>({c, std::min<int64_t>(slice_cluster, kMaxCluster),
                             std::max<int64_t>(1, ceil_div(row_stride, kSliceMinElems))});
      c = std::max(c, cmin);
      while (c > cmin && !fits(c)) --c;
      const int64_t ch = slice_chunks(row_stride, c, eb);
      const int64_t lcap = slice_list_cap(ch, smem_optin, eb);
      const SliceLayout sl = slice_layout(ch, lcap, eb);
      p.kernel = DSEL_KERNEL_SLICE;
      p.threads = slice_threads(ch);
      p.cluster = int(c);
      p.groups = 1;
      p.stages = int(ch);
      p.block = kSliceChunkBytes / eb;
      p.round = int(round_up(ceil_div(row_stride, c), 16));
      p.b2 = 0;
      p.capacity = int(lcap);
      p.idx_bits = ceil_log2_u64(uint64_t(row_stride));
      p.smem_bytes = int(sl.total);
      p.workspace_bytes = 0;
      *out = p;
      return DSEL_OK;
    }
  }
  const bool short_rows = one_per_row && row_stride <= 2 * int64_t(round_elems(dtype, kThreadsShort));

  // 256-thread shape: two CTAs per SM (half of the SM's shared memory each, less
  // the 1 KB the hardware reserves per CTA) with at least one round in flight
  int64_t mid_stages = 0;
  if (one_per_row && !short_rows && k <= 1024) {
    dsel_plan_t m{};
    shape_plan(dtype, k, kThreadsMid, &m);
    const int64_t budget = (int64_t(smem_optin) + 1024) / 2 - 1024;
    const int64_t nb = ceil_div(row_stride, m.block);
    const int64_t q = m.round / m.block;
    for (int64_t s = std::min<int64_t>(nb, 2 * q); s >= std::min<int64_t>(nb, q); --s) {
      if ((s == nb || s % q == 0) && shape_smem(m, s, k, eb) <= budget) {
        mid_stages = s;
        break;
      }
    }
  }
  p.kernel = DSEL_KERNEL_STREAM;
  shape_plan(dtype, k, short_rows ? kThreadsShort : (mid_stages > 0 ? kThreadsMid : kThreads), &p);
  p.idx_bits = ceil_log2_u64(uint64_t(row_stride));

  // Row split.
  int64_t splits = 1;
  if (!one_per_row) {
    splits = num_sms / std::max<int64_t>(rows, 1);
    splits = std::min<int64_t>(splits, std::max<int64_t>(1, row_stride / kMinSliceElems));
    splits = std::max<int64_t>(splits, 1);
  }
  int64_t cluster = std::min<int64_t>(splits, max_cluster);
  int64_t groups = std::max<int64_t>(1, splits / cluster);
  // the merge holds all groups' partial results across at most kMaxCluster CTAs
  const int64_t max_groups =
      std::min<int64_t>(kMaxGroups, std::max<int64_t>(1, int64_t(kMaxCluster) * p.capacity / k));
  groups = std::min(groups, max_groups);
  // On a device whose cluster capacity is known: the split with the most CTAs
  // whose clusters the device holds all at once (non-portable sizes included),
  // fewer groups first among equals.  A launch whose clusters need two waves
  // takes about twice as long: sixteen rows of 2^24 f32 ran in 1,064 us in
  // clusters of 8 (one group) and in 613 us in clusters of 4 (two groups).
  if (cluster_fit != nullptr && splits > 1) {
    int64_t bc = 0, bg = 0;
    const int64_t cmax = std::min<int64_t>(splits, kSliceMaxCluster);
    for (int64_t c = 2; c <= cmax; ++c) {
      if (cluster_fit[c] < 1) continue;
      int64_t g = std::min<int64_t>(std::max<int64_t>(1, splits / c), max_groups);
      if (rows * g > cluster_fit[c]) g = cluster_fit[c] / rows;
      if (g < 1) continue;
      if (c * g > bc * bg || (c * g == bc * bg && g < bg)) {
        bc = c;
        bg = g;
      }
    }
    if (bc > 0) {
      cluster = bc;
      groups = bg;
    }
  }
  p.cluster = int(cluster);
  p.groups = int(groups);

  // Ring depth.
  const int64_t slice = round_up(ceil_div(row_stride, groups * cluster), kStrideReq);
  const int64_t nb_max = ceil_div(slice, p.block);
  const int64_t per_round = p.round / p.block;
  const int64_t base = shape_smem(p, 0, k, eb) + 256;
  const int64_t per_stage = int64_t(p.block) * eb + 8 + 4;
  int64_t stages = (int64_t(smem_optin) - base) / per_stage;
  stages = std::min<int64_t>(stages, kMaxStages);
  if (short_rows) {
    stages = std::min(nb_max, per_round);    // one round in flight: keeps several CTAs per SM
  } else if (mid_stages > 0) {
    stages = mid_stages;                     // two CTAs per SM
  } else if (nb_max <= stages) {
    stages = nb_max;                         // the whole slice in flight at once, no refills
  } else {
    stages = stages / per_round * per_round; // refills go to the warp that owns the stage
  }
  stages = std::max<int64_t>(stages, std::min<int64_t>(per_round, nb_max));
  p.stages = int(stages);
  const int64_t smem = shape_smem(p, stages, k, eb);
  if (smem > smem_optin) return DSEL_ERR_K;
  p.smem_bytes = int(smem);

  // Split-row workspace: each cluster leaves up to k (bits, index) pairs and a
  // (count, flags) word per row.
  p.workspace_bytes = groups > 1 ? rows * groups * (int64_t(k) * 8 + 8) : 0;
  *out = p;
  return DSEL_OK;
}

}  // namespace dsel
