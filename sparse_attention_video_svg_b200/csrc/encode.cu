// Mask encodings and the energy-threshold schedule.
//
// CalibAtt article (lpnh.cn/news/568491), section 3.1: the energy threshold
// eps(t) decays exponentially over the denoising steps, about 0.99 early and
// 0.84 late; section 3.3: the sparse mask is precomputed as a skip list of
// contiguous block intervals, and stored as a bitmap that takes 32x less
// memory.
//
//   svg_epsilon_schedule    host: eps_i = first * (last / first)^(i / (n - 1))
//   svg_lists_to_intervals  CSR lists -> maximal runs [start, end) per row
//                           (count pass, scan, fill; warp per row)
//   svg_lists_to_bitmap     CSR lists -> one bit per (row, block) in 32-bit
//                           words (warp per row)
#include <math.h>

#include "common.cuh"

namespace svg {
namespace {

constexpr int kRowsPerBlock = 8;  // one warp per row
constexpr int kScanThreads = 1024;

// Entries [b, e) of row r, or an empty range (flagged) for a bad indptr.
__device__ __forceinline__ bool row_range(const int32_t* indptr, int r, int& b, int& e,
                                          int32_t* status) {
  b = indptr[r];
  e = indptr[r + 1];
  if (b < 0 || e < b) {
    if ((threadIdx.x & 31) == 0) set_status(status, SVG_DEVICE_BAD_INDEX);
    b = e = 0;
    return false;
  }
  return true;
}

// Does entry t of the row start a new run?  A run continues while the next
// index is the same block (a duplicate) or the next one.
__device__ __forceinline__ bool starts_run(const int32_t* idx, int b, int t) {
  if (t == b) return true;
  const int prev = idx[t - 1], c = idx[t];
  return !(c == prev || c == prev + 1);
}

__device__ __forceinline__ bool ends_run(const int32_t* idx, int e, int t) {
  if (t + 1 == e) return true;
  const int c = idx[t], next = idx[t + 1];
  return !(next == c || next == c + 1);
}

// counts[r + 1] = runs in row r; flags indices outside [0, n_cols) and rows
// that are not ascending.
__global__ void interval_count_kernel(int n_rows, int n_cols, const int32_t* __restrict__ indptr,
                                      const int32_t* __restrict__ idx, int32_t* __restrict__ iptr,
                                      int32_t* status) {
  const int r = blockIdx.x * kRowsPerBlock + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (r >= n_rows) return;
  if (r == 0 && lane == 0) iptr[0] = 0;
  int b, e;
  row_range(indptr, r, b, e, status);
  int runs = 0;
  bool bad = false;
  for (int t = b + lane; t < e; t += 32) {
    const int c = idx[t];
    bad |= c < 0 || c >= n_cols || (t > b && c < idx[t - 1]);
    runs += starts_run(idx, b, t) ? 1 : 0;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) runs += __shfl_xor_sync(0xffffffffu, runs, o);
  if (__any_sync(0xffffffffu, bad) && lane == 0) set_status(status, SVG_DEVICE_BAD_INDEX);
  if (lane == 0) iptr[r + 1] = runs;
}

// In-place inclusive scan of iptr[1 .. n_rows] (one CTA); the total goes to
// n_out.
__global__ void __launch_bounds__(kScanThreads) interval_scan_kernel(int n_rows,
                                                                     int32_t* __restrict__ iptr,
                                                                     int64_t* __restrict__ n_out) {
  __shared__ long long part[kScanThreads];
  __shared__ long long carry;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < n_rows; base += kScanThreads) {
    const int i = base + threadIdx.x;
    long long x = i < n_rows ? iptr[i + 1] : 0;
    part[threadIdx.x] = x;
    __syncthreads();
    for (int off = 1; off < kScanThreads; off <<= 1) {
      const long long y = threadIdx.x >= off ? part[threadIdx.x - off] : 0;
      __syncthreads();
      part[threadIdx.x] += y;
      __syncthreads();
    }
    if (i < n_rows) iptr[i + 1] = static_cast<int32_t>(carry + part[threadIdx.x]);
    __syncthreads();
    if (threadIdx.x == 0) carry += part[kScanThreads - 1];
    __syncthreads();
  }
  if (threadIdx.x == 0 && n_out != nullptr) *n_out = carry;
}

// starts / ends of every run, at the row's offset iptr[r]; runs past
// `capacity` are not written (SVG_DEVICE_CAPACITY).
__global__ void interval_fill_kernel(int n_rows, const int32_t* __restrict__ indptr,
                                     const int32_t* __restrict__ idx,
                                     const int32_t* __restrict__ iptr, int32_t* __restrict__ starts,
                                     int32_t* __restrict__ ends, long long capacity,
                                     int32_t* status) {
  const int r = blockIdx.x * kRowsPerBlock + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (r >= n_rows) return;
  int b, e;
  if (!row_range(indptr, r, b, e, nullptr)) return;
  long long out = iptr[r];  // next run slot of this row
  bool over = false;
  for (int t0 = b; t0 < e; t0 += 32) {
    const int t = t0 + lane;
    const bool s = t < e && starts_run(idx, b, t);
    const bool f = t < e && ends_run(idx, e, t);
    const unsigned sm = __ballot_sync(0xffffffffu, s);
    const unsigned fm = __ballot_sync(0xffffffffu, f);
    // the k-th start of this chunk is run out + k; an end belongs to the run
    // opened by the latest start at or before it (possibly in an earlier
    // chunk: then it is run out - 1)
    if (s) {
      const long long slot = out + __popc(sm & ((1u << lane) - 1u));
      if (slot < capacity) starts[slot] = idx[t];
      else over = true;
    }
    if (f) {
      const long long slot = out + __popc(sm & ((2u << lane) - 1u)) - 1;
      if (slot < capacity) ends[slot] = idx[t] + 1;
      else over = true;
    }
    out += __popc(sm);
    (void)fm;
  }
  if (__any_sync(0xffffffffu, over) && lane == 0) set_status(status, SVG_DEVICE_CAPACITY);
}

// One bit per kept block: the row's words are cleared, then each index sets
// its bit.
__global__ void bitmap_kernel(int n_rows, int n_cols, const int32_t* __restrict__ indptr,
                              const int32_t* __restrict__ idx, uint32_t* __restrict__ bitmap,
                              int32_t* status) {
  const int r = blockIdx.x * kRowsPerBlock + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (r >= n_rows) return;
  const int words = (n_cols + 31) / 32;
  uint32_t* row = bitmap + static_cast<long long>(r) * words;
  for (int w = lane; w < words; w += 32) row[w] = 0u;
  __syncwarp();
  int b, e;
  row_range(indptr, r, b, e, status);
  bool bad = false;
  for (int t = b + lane; t < e; t += 32) {
    const int c = idx[t];
    if (c < 0 || c >= n_cols) {
      bad = true;
      continue;
    }
    atomicOr(&row[c >> 5], 1u << (c & 31));
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) set_status(status, SVG_DEVICE_BAD_INDEX);
}

}  // namespace
}  // namespace svg

using namespace svg;

extern "C" svg_status svg_epsilon_schedule(int n_steps, double eps_first, double eps_last,
                                           double* eps_out) {
  clear_error();
  if (n_steps < 0 || (n_steps > 0 && eps_out == nullptr))
    return fail(SVG_ERR_INVALID_ARG, "epsilon_schedule: bad n_steps or null output");
  if (!(eps_first > 0.0 && eps_first <= 1.0 && eps_last > 0.0 && eps_last <= 1.0))
    return fail(SVG_ERR_INVALID_ARG, "epsilon_schedule: thresholds must lie in (0, 1]");
  for (int i = 0; i < n_steps; ++i)
    eps_out[i] = n_steps == 1 ? eps_first
                              : eps_first * pow(eps_last / eps_first,
                                                static_cast<double>(i) / (n_steps - 1));
  return SVG_OK;
}

extern "C" svg_status svg_lists_to_intervals(int n_rows, int n_cols, const int32_t* indptr,
                                             const int32_t* indices, int32_t* iptr,
                                             int32_t* starts, int32_t* ends, int64_t capacity,
                                             int64_t* n_out, int32_t* device_status,
                                             void* stream) {
  clear_error();
  if (n_rows <= 0 || n_cols <= 0 || capacity < 0)
    return fail(SVG_ERR_INVALID_ARG, "lists_to_intervals: bad sizes");
  if (indptr == nullptr || indices == nullptr || iptr == nullptr)
    return fail(SVG_ERR_INVALID_ARG, "lists_to_intervals: null pointer");
  if (capacity > 0 && (starts == nullptr || ends == nullptr))
    return fail(SVG_ERR_INVALID_ARG, "lists_to_intervals: null starts / ends");
  cudaStream_t s = as_stream(stream);
  const int blocks = (n_rows + kRowsPerBlock - 1) / kRowsPerBlock;
  interval_count_kernel<<<blocks, 32 * kRowsPerBlock, 0, s>>>(n_rows, n_cols, indptr, indices,
                                                              iptr, device_status);
  if (svg_status st = check_launch("lists_to_intervals count")) return st;
  interval_scan_kernel<<<1, kScanThreads, 0, s>>>(n_rows, iptr, n_out);
  if (svg_status st = check_launch("lists_to_intervals scan")) return st;
  if (capacity == 0) return SVG_OK;  // size query
  interval_fill_kernel<<<blocks, 32 * kRowsPerBlock, 0, s>>>(
      n_rows, indptr, indices, iptr, starts, ends, capacity, device_status);
  return check_launch("lists_to_intervals fill");
}

extern "C" svg_status svg_lists_to_bitmap(int n_rows, int n_cols, const int32_t* indptr,
                                          const int32_t* indices, uint32_t* bitmap,
                                          int32_t* device_status, void* stream) {
  clear_error();
  if (n_rows <= 0 || n_cols <= 0) return fail(SVG_ERR_INVALID_ARG, "lists_to_bitmap: bad sizes");
  if (indptr == nullptr || indices == nullptr || bitmap == nullptr)
    return fail(SVG_ERR_INVALID_ARG, "lists_to_bitmap: null pointer");
  const int blocks = (n_rows + kRowsPerBlock - 1) / kRowsPerBlock;
  bitmap_kernel<<<blocks, 32 * kRowsPerBlock, 0, as_stream(stream)>>>(n_rows, n_cols, indptr,
                                                                      indices, bitmap,
                                                                      device_status);
  return check_launch("lists_to_bitmap");
}
