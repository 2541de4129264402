// Row split over several shards (one per GPU): the re-layout of the gathered
// per-shard candidates and the index map back to the whole row.  Both are
// plain elementwise kernels (HBM-bound, a few KB to a few MB per call): one
// thread per output element, consecutive threads on consecutive columns.
#include <cstdint>

#include <cuda_runtime.h>

#include "dsel_plan.h"   // the C ABI (include/dsel.h) and the shape limits

namespace dsel {
namespace {

constexpr int kEltThreads = 256;

template <typename bits_t>
__global__ void __launch_bounds__(kEltThreads) shard_stack_kernel(const bits_t* __restrict__ vals_in,
                                                                  const int64_t* __restrict__ idx_in, int64_t rows,
                                                                  int32_t k, int32_t shards, int64_t shard_len,
                                                                  int64_t out_stride, bits_t neg_inf,
                                                                  bits_t* __restrict__ vals_out,
                                                                  int64_t* __restrict__ idx_out) {
  const int64_t total = rows * out_stride;
  const int64_t width = static_cast<int64_t>(shards) * k;
  for (int64_t o = static_cast<int64_t>(blockIdx.x) * kEltThreads + threadIdx.x; o < total;
       o += static_cast<int64_t>(gridDim.x) * kEltThreads) {
    const int64_t r = o / out_stride, c = o - r * out_stride;
    if (c < width) {
      const int64_t s = c / k, j = c - s * k;
      const int64_t src = (s * rows + r) * k + j;
      const int64_t idx = idx_in[src];
      vals_out[o] = vals_in[src];
      idx_out[o] = idx >= 0 ? idx + s * shard_len : idx;
    } else {
      vals_out[o] = neg_inf;
      idx_out[o] = DSEL_IDX_PAD;
    }
  }
}

template <typename pos_t, typename out_t>
__global__ void __launch_bounds__(kEltThreads) take_index_kernel(const int64_t* __restrict__ table,
                                                                 int64_t table_stride, const pos_t* __restrict__ pos,
                                                                 int64_t rows, int32_t k, out_t* __restrict__ out) {
  const int64_t total = rows * k;
  for (int64_t o = static_cast<int64_t>(blockIdx.x) * kEltThreads + threadIdx.x; o < total;
       o += static_cast<int64_t>(gridDim.x) * kEltThreads) {
    const int64_t r = o / k;
    const int64_t p = static_cast<int64_t>(pos[o]);
    out[o] = static_cast<out_t>(p >= 0 ? table[r * table_stride + p] : p);
  }
}

unsigned grid_for(int64_t total) {
  const int64_t blocks = (total + kEltThreads - 1) / kEltThreads;
  const int64_t cap = 148 * 16;   // grid-stride beyond a few waves of the 148 SMs
  return static_cast<unsigned>(blocks < cap ? (blocks > 0 ? blocks : 1) : cap);
}

}  // namespace
}  // namespace dsel

using namespace dsel;

DSEL_API int dsel_shard_stack(const void* vals_in, const int64_t* idx_in, int dtype, int64_t rows, int32_t k,
                              int32_t shards, int64_t shard_len, int64_t out_stride, void* vals_out,
                              int64_t* idx_out, void* stream) {
  if (dtype != DSEL_BF16 && dtype != DSEL_F32) return DSEL_ERR_DTYPE;
  if (k < 1 || k > kMaxK || shards < 1 || shard_len < k) return DSEL_ERR_K;
  if (rows < 0) return DSEL_ERR_ROWS;
  if (out_stride < static_cast<int64_t>(shards) * k || out_stride % kStrideReq != 0 || out_stride > INT32_MAX)
    return DSEL_ERR_STRIDE;
  if (rows == 0) return DSEL_OK;
  if (vals_in == nullptr || idx_in == nullptr || vals_out == nullptr || idx_out == nullptr) return DSEL_ERR_NULL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const unsigned grid = grid_for(rows * out_stride);
  if (dtype == DSEL_BF16)
    shard_stack_kernel<uint16_t><<<grid, kEltThreads, 0, st>>>(
        static_cast<const uint16_t*>(vals_in), idx_in, rows, k, shards, shard_len, out_stride,
        static_cast<uint16_t>(0xFF80u), static_cast<uint16_t*>(vals_out), idx_out);
  else
    shard_stack_kernel<uint32_t><<<grid, kEltThreads, 0, st>>>(
        static_cast<const uint32_t*>(vals_in), idx_in, rows, k, shards, shard_len, out_stride, 0xFF800000u,
        static_cast<uint32_t*>(vals_out), idx_out);
  return cudaGetLastError() == cudaSuccess ? DSEL_OK : DSEL_ERR_CUDA;
}

DSEL_API int dsel_take_index(const int64_t* table, int64_t table_stride, const void* pos, int pos_dtype, int64_t rows,
                             int32_t k, int index_dtype, void* indices_out, void* stream) {
  if (k < 1 || k > kMaxK || table_stride < 1) return DSEL_ERR_K;
  if (rows < 0) return DSEL_ERR_ROWS;
  if ((pos_dtype != DSEL_I32 && pos_dtype != DSEL_I64) || (index_dtype != DSEL_I32 && index_dtype != DSEL_I64))
    return DSEL_ERR_INDEX_DTYPE;
  if (rows == 0) return DSEL_OK;
  if (table == nullptr || pos == nullptr || indices_out == nullptr) return DSEL_ERR_NULL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const unsigned grid = grid_for(rows * k);
  if (pos_dtype == DSEL_I32) {
    if (index_dtype == DSEL_I32)
      take_index_kernel<int32_t, int32_t><<<grid, kEltThreads, 0, st>>>(
          table, table_stride, static_cast<const int32_t*>(pos), rows, k, static_cast<int32_t*>(indices_out));
    else
      take_index_kernel<int32_t, int64_t><<<grid, kEltThreads, 0, st>>>(
          table, table_stride, static_cast<const int32_t*>(pos), rows, k, static_cast<int64_t*>(indices_out));
  } else {
    if (index_dtype == DSEL_I32)
      take_index_kernel<int64_t, int32_t><<<grid, kEltThreads, 0, st>>>(
          table, table_stride, static_cast<const int64_t*>(pos), rows, k, static_cast<int32_t*>(indices_out));
    else
      take_index_kernel<int64_t, int64_t><<<grid, kEltThreads, 0, st>>>(
          table, table_stride, static_cast<const int64_t*>(pos), rows, k, static_cast<int64_t*>(indices_out));
  }
  return cudaGetLastError() == cudaSuccess ? DSEL_OK : DSEL_ERR_CUDA;
}
