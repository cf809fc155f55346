// Per-query-block key-block lists (CSR) for block-sparse attention.
//
// CalibAtt article (lpnh.cn/news/568491): section 2.2 makes keep/skip decisions
// on 128x128 tiles; section 3.1 keeps, per query block, the shortest
// descending-energy prefix of key blocks reaching eps and votes across inputs
// with threshold rho; section 3.3 encodes the result as a per-row skip list.
// Sparse VideoGen article (m.jxzklqfsx.com/article/815093.html), sections
// "Spatial Head" and "Temporal Head", give the two geometric token masks.
//
// Geometric lists.  The frames (spatial, frame-major) or positions (temporal,
// token-major) of tile j's tokens form the interval [lo_j, hi_j] with lo, hi
// non-decreasing in j, so the key tiles that meet query tile i's band form
// one contiguous run [J0, J1]:
//     J0 = first tile holding token (lo_i - w) * div   (0 if lo_i - w <= 0)
//     J1 = tile holding the last token of frame/position hi_i + w (clipped)
// with div = P, w = spatial_width (spatial) or div = F, w = 0 (temporal).
#include <float.h>

#include "common.cuh"

namespace svg {
namespace {

constexpr int kScanThreads = 1024;

struct GeoRow {
  int j0, j1;
};

__device__ __forceinline__ GeoRow geo_row(int kind, int i, int nb, int N, int div, int w) {
  if (kind == SVG_MODE_DENSE) return {0, nb - 1};
  const long long T = SVG_TILE;
  const long long lo = (i * T) / div;
  const long long last = (i + 1) * T < N ? (i + 1) * T - 1 : N - 1;
  const long long hi = last / div;
  const long long L = lo - w;
  const long long U = hi + w;
  long long j0 = L > 0 ? (L * div) / T : 0;
  long long j1 = ((U + 1) * div - 1) / T;
  if (j1 > nb - 1) j1 = nb - 1;
  return {static_cast<int>(j0), static_cast<int>(j1)};
}

// Block-wide inclusive scan of one int per thread (kScanThreads threads).
__device__ __forceinline__ long long block_inclusive_scan(long long x, long long* warp_sums) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    long long y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    long long s = lane < (kScanThreads / 32) ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      long long y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    warp_sums[lane] = s;
  }
  __syncthreads();
  if (warp > 0) x += warp_sums[warp - 1];
  return x;
}

// One block: row counts of the geometric lists, scanned into indptr; nnz.
__global__ void __launch_bounds__(kScanThreads) geo_scan_kernel(int kind, int N, int nb, int div,
                                                                int w, int base_off,
                                                                int32_t* indptr,
                                                                int64_t* nnz_out) {
  __shared__ long long warp_sums[32];
  __shared__ long long carry_s;
  if (threadIdx.x == 0) {
    carry_s = 0;
    indptr[0] = base_off;
  }
  __syncthreads();
  for (int base = 0; base < nb; base += kScanThreads) {
    const int i = base + threadIdx.x;
    long long cnt = 0;
    if (i < nb) {
      GeoRow r = geo_row(kind, i, nb, N, div, w);
      cnt = r.j1 - r.j0 + 1;
    }
    const long long carry = carry_s;
    const long long incl = block_inclusive_scan(cnt, warp_sums);
    if (i < nb) indptr[i + 1] = static_cast<int32_t>(base_off + carry + incl);
    __syncthreads();
    if (threadIdx.x == kScanThreads - 1) carry_s = carry + incl;
    __syncthreads();
  }
  if (threadIdx.x == 0) *nnz_out = carry_s;
}

// One warp per query tile: writes J0..J1.
__global__ void geo_fill_kernel(int kind, int N, int nb, int div, int w, int base_off,
                                const int32_t* __restrict__ indptr, int32_t* __restrict__ indices,
                                int64_t capacity, const int64_t* __restrict__ nnz,
                                int32_t* status) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= nb) return;
  if (*nnz > capacity) {
    if (warp == 0 && lane == 0) set_status(status, SVG_DEVICE_CAPACITY);
    return;
  }
  GeoRow r = geo_row(kind, warp, nb, N, div, w);
  const int off = indptr[warp] - base_off;
  for (int j = r.j0 + lane; j <= r.j1; j += 32) indices[off + (j - r.j0)] = j;
}

// ------------------------------------------------------------ calibrated lists

constexpr int kCalThreads = 512;
constexpr int kMaxKB = 4096;
constexpr int kMaxR = 16;

// Order-preserving map of a float to uint32 (larger float -> larger code).
__device__ __forceinline__ uint32_t float_order(float f) {
  const uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// One block per (list, query block): sort, cut at eps for every input, vote,
// and write the kept set as a bitmap plus its count.
__global__ void __launch_bounds__(kCalThreads) calib_rows_kernel(
    const float* __restrict__ energy, int R, int rows, int nKB, int npow2, double eps,
    double rho, uint32_t* __restrict__ bitmap, int32_t* __restrict__ counts) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  unsigned long long* keys = reinterpret_cast<unsigned long long*>(smem_raw);  // [npow2]
  float* e = reinterpret_cast<float*>(keys + npow2);                          // [nKB]
  int* votes = reinterpret_cast<int*>(e + nKB);                               // [nKB]
  __shared__ int any_kept;
  __shared__ double best_val[kCalThreads / 32];
  __shared__ int best_idx[kCalThreads / 32];

  const int row = blockIdx.x;  // = list * nQB + query block
  const long long row_stride = static_cast<long long>(rows) * nKB;
  for (int c = threadIdx.x; c < nKB; c += blockDim.x) votes[c] = 0;

  for (int s = 0; s < R; ++s) {
    const float* src = energy + s * row_stride + static_cast<long long>(row) * nKB;
    __syncthreads();
    for (int c = threadIdx.x; c < npow2; c += blockDim.x) {
      if (c < nKB) {
        const float v = src[c];
        e[c] = v;
        // ascending key order = descending energy, then ascending index
        keys[c] = (static_cast<unsigned long long>(~float_order(v)) << 32) | static_cast<uint32_t>(c);
      } else {
        keys[c] = ~0ull;
      }
    }
    __syncthreads();
    // bitonic sort, ascending
    for (int k = 2; k <= npow2; k <<= 1) {
      for (int j = k >> 1; j > 0; j >>= 1) {
        for (int t = threadIdx.x; t < npow2; t += blockDim.x) {
          const int p = t ^ j;
          if (p > t) {
            const unsigned long long a = keys[t], b = keys[p];
            const bool up = (t & k) == 0;
            if ((a > b) == up) {
              keys[t] = b;
              keys[p] = a;
            }
          }
        }
        __syncthreads();
      }
    }
    // the running sum must follow the sorted order exactly: one thread
    if (threadIdx.x == 0) {
      double acc = 0.0;
      for (int t = 0; t < nKB; ++t) {
        const int c = static_cast<int>(keys[t] & 0xffffffffu);
        votes[c] += 1;
        acc += static_cast<double>(e[c]);
        if (acc >= eps) break;
      }
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) any_kept = 0;
  __syncthreads();
  const int words = (nKB + 31) / 32;
  uint32_t* bm = bitmap + static_cast<long long>(row) * words;
  int local = 0;
  for (int wd = threadIdx.x; wd < words; wd += blockDim.x) {
    uint32_t bits = 0;
    for (int b = 0; b < 32; ++b) {
      const int c = wd * 32 + b;
      if (c < nKB && static_cast<double>(votes[c]) / static_cast<double>(R) >= rho) bits |= 1u << b;
    }
    bm[wd] = bits;
    local += __popc(bits);
  }
  if (local) atomicAdd(&any_kept, local);
  __syncthreads();
  if (any_kept == 0) {
    // fallback: argmax of the energy summed over inputs (in input order)
    double bv = -DBL_MAX;
    int bi = 0x7fffffff;
    for (int c = threadIdx.x; c < nKB; c += blockDim.x) {
      double tot = 0.0;
      for (int s = 0; s < R; ++s)
        tot = tot + static_cast<double>(energy[s * row_stride + static_cast<long long>(row) * nKB + c]);
      if (tot > bv || (tot == bv && c < bi)) {
        bv = tot;
        bi = c;
      }
    }
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const double ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) {
        bv = ov;
        bi = oi;
      }
    }
    if (lane == 0) {
      best_val[warp] = bv;
      best_idx[warp] = bi;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      for (int wI = 1; wI < static_cast<int>(blockDim.x / 32); ++wI)
        if (best_val[wI] > bv || (best_val[wI] == bv && best_idx[wI] < bi)) {
          bv = best_val[wI];
          bi = best_idx[wI];
        }
      bm[bi / 32] |= 1u << (bi % 32);
      counts[row] = 1;
    }
  } else if (threadIdx.x == 0) {
    counts[row] = any_kept;
  }
}

// One block: scan the per-row counts into the [L][nQB + 1] indptr layout.
__global__ void __launch_bounds__(kScanThreads) calib_scan_kernel(const int32_t* __restrict__ counts,
                                                                  int L, int nQB, int32_t* indptr,
                                                                  int64_t* nnz_out) {
  __shared__ long long warp_sums[32];
  __shared__ long long carry_s;
  if (threadIdx.x == 0) carry_s = 0;
  __syncthreads();
  const int rows = L * nQB;
  for (int base = 0; base < rows; base += kScanThreads) {
    const int g = base + threadIdx.x;
    const long long cnt = g < rows ? counts[g] : 0;
    const long long carry = carry_s;
    const long long incl = block_inclusive_scan(cnt, warp_sums);
    if (g < rows) {
      const int l = g / nQB, i = g - l * nQB;
      if (i == 0) indptr[l * (nQB + 1)] = static_cast<int32_t>(carry + incl - cnt);
      indptr[l * (nQB + 1) + i + 1] = static_cast<int32_t>(carry + incl);
    }
    __syncthreads();
    if (threadIdx.x == kScanThreads - 1) carry_s = carry + incl;
    __syncthreads();
  }
  if (threadIdx.x == 0) *nnz_out = carry_s;
}

// One warp per row: bitmap -> ascending indices.
__global__ void calib_fill_kernel(const uint32_t* __restrict__ bitmap, int L, int nQB, int nKB,
                                  const int32_t* __restrict__ indptr, int32_t* __restrict__ indices,
                                  int64_t capacity, const int64_t* __restrict__ nnz,
                                  int32_t* status) {
  const int g = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (g >= L * nQB) return;
  if (*nnz > capacity) {
    if (g == 0 && lane == 0) set_status(status, SVG_DEVICE_CAPACITY);
    return;
  }
  const int l = g / nQB, i = g - l * nQB;
  int off = indptr[l * (nQB + 1) + i];
  const int words = (nKB + 31) / 32;
  const uint32_t* bm = bitmap + static_cast<long long>(g) * words;
  for (int wd = 0; wd < words; ++wd) {
    const uint32_t bits = bm[wd];
    const bool mine = (bits >> lane) & 1u;
    const int before = __popc(bits & ((1u << lane) - 1u));
    if (mine) indices[off + before] = wd * 32 + lane;
    off += __popc(bits);
  }
}

}  // namespace
}  // namespace svg

using namespace svg;

extern "C" svg_status svg_build_block_mask(int kind, int frames, int tokens_per_frame,
                                           int spatial_width, int N, int32_t* indptr,
                                           int32_t* indices, int64_t capacity,
                                           int64_t index_base, int64_t* nnz_out,
                                           int32_t* device_status, void* stream) {
  clear_error();
  if (kind != SVG_MODE_SPATIAL && kind != SVG_MODE_TEMPORAL && kind != SVG_MODE_DENSE)
    return fail(SVG_ERR_INVALID_ARG, "build_block_mask: bad kind %d", kind);
  if (frames <= 0 || tokens_per_frame <= 0 || N <= 0 ||
      static_cast<long long>(frames) * tokens_per_frame != N)
    return fail(SVG_ERR_INVALID_ARG, "build_block_mask: frames*tokens_per_frame != N");
  if (spatial_width < 0) return fail(SVG_ERR_INVALID_ARG, "build_block_mask: spatial_width < 0");
  if (indptr == nullptr || nnz_out == nullptr || (indices == nullptr && capacity > 0) ||
      capacity < 0)
    return fail(SVG_ERR_INVALID_ARG, "build_block_mask: null output");
  const int nb = n_tiles(N);
  if (index_base < 0 || static_cast<long long>(nb) * nb + index_base > 0x7fffffffLL)
    return fail(SVG_ERR_UNSUPPORTED, "build_block_mask: offsets exceed int32 (index_base %lld)",
                static_cast<long long>(index_base));
  const int base_off = static_cast<int>(index_base);
  const int div = kind == SVG_MODE_TEMPORAL ? frames : tokens_per_frame;
  const int w = kind == SVG_MODE_SPATIAL ? spatial_width : 0;
  cudaStream_t s = as_stream(stream);
  geo_scan_kernel<<<1, kScanThreads, 0, s>>>(kind, N, nb, div, w, base_off, indptr, nnz_out);
  if (svg_status st = check_launch("build_block_mask scan")) return st;
  const int warps_per_block = 8;
  geo_fill_kernel<<<(nb + warps_per_block - 1) / warps_per_block, 32 * warps_per_block, 0, s>>>(
      kind, N, nb, div, w, base_off, indptr, indices, capacity, nnz_out, device_status);
  return check_launch("build_block_mask fill");
}

extern "C" size_t svg_calibrated_workspace_size(int L, int nQB, int nKB) {
  if (L <= 0 || nQB <= 0 || nKB <= 0) return 0;
  const size_t words = (static_cast<size_t>(nKB) + 31) / 32;
  const size_t bitmap = static_cast<size_t>(L) * nQB * words * 4;
  const size_t counts = static_cast<size_t>(L) * nQB * 4;
  return ((bitmap + 255) / 256) * 256 + ((counts + 255) / 256) * 256;
}

extern "C" svg_status svg_build_block_mask_calibrated(const float* energy, int R, int L, int nQB,
                                                      int nKB, double eps, double rho,
                                                      int32_t* indptr, int32_t* indices,
                                                      int64_t capacity, int64_t* nnz_out,
                                                      int32_t* device_status, void* workspace,
                                                      size_t workspace_bytes, void* stream) {
  clear_error();
  if (energy == nullptr || indptr == nullptr || nnz_out == nullptr || workspace == nullptr ||
      (indices == nullptr && capacity > 0) || capacity < 0)
    return fail(SVG_ERR_INVALID_ARG, "calibrated: null pointer");
  if (R < 1 || R > kMaxR) return fail(SVG_ERR_INVALID_ARG, "calibrated: R=%d not in [1,%d]", R, kMaxR);
  if (L <= 0 || nQB <= 0 || nKB <= 0 || nKB > kMaxKB)
    return fail(SVG_ERR_INVALID_ARG, "calibrated: bad L=%d nQB=%d nKB=%d (nKB <= %d)", L, nQB, nKB,
                kMaxKB);
  if (!(eps > 0.0) || !(rho >= 0.0) || rho > 1.0)
    return fail(SVG_ERR_INVALID_ARG, "calibrated: need eps > 0 and 0 <= rho <= 1");
  if (static_cast<long long>(L) * nQB * nKB > 0x7fffffffLL)
    return fail(SVG_ERR_UNSUPPORTED, "calibrated: too many entries for int32 offsets");
  if (workspace_bytes < svg_calibrated_workspace_size(L, nQB, nKB) || !aligned256(workspace))
    return fail(SVG_ERR_INVALID_ARG, "calibrated: workspace too small or not 256-byte aligned");
  const size_t words = (static_cast<size_t>(nKB) + 31) / 32;
  const size_t bitmap_bytes = ((static_cast<size_t>(L) * nQB * words * 4 + 255) / 256) * 256;
  auto* bitmap = static_cast<uint32_t*>(workspace);
  auto* counts = reinterpret_cast<int32_t*>(static_cast<char*>(workspace) + bitmap_bytes);
  int npow2 = 1;
  while (npow2 < nKB) npow2 <<= 1;
  const size_t smem = static_cast<size_t>(npow2) * 8 + static_cast<size_t>(nKB) * 8;
  cudaStream_t s = as_stream(stream);
  if (smem > 48 * 1024) {
    if (cudaFuncSetAttribute(calib_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return fail(SVG_ERR_CUDA, "calibrated: cannot reserve %zu bytes of shared memory", smem);
  }
  const int rows = L * nQB;
  calib_rows_kernel<<<rows, kCalThreads, smem, s>>>(energy, R, rows, nKB, npow2, eps, rho, bitmap,
                                                    counts);
  if (svg_status st = check_launch("calibrated rows")) return st;
  calib_scan_kernel<<<1, kScanThreads, 0, s>>>(counts, L, nQB, indptr, nnz_out);
  if (svg_status st = check_launch("calibrated scan")) return st;
  calib_fill_kernel<<<(rows + 7) / 8, 256, 0, s>>>(bitmap, L, nQB, nKB, indptr, indices, capacity,
                                                   nnz_out, device_status);
  return check_launch("calibrated fill");
}
