// Frame-major <-> token-major permutation of [B, H, N, d] tensors.
//
// Sparse VideoGen article (m.jxzklqfsx.com/article/815093.html), section
// "Layout Transformation + Kernel 加速": a temporal head needs one spatial
// position in every frame; in frame-major order (n = f P + s) those tokens are
// P rows apart, in token-major order (m = s F + f) they are adjacent.
//
// Each token row is d * elt = 128-512 contiguous bytes, so the permutation is a
// row gather: threads walk the DESTINATION in order (fully coalesced stores)
// and read each source row as whole 16-byte chunks (every 32-byte sector read
// is used).  No shared-memory transpose is needed.  HBM-bound: 2 N d elt bytes
// per head.
#include "common.cuh"

namespace svg {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;  // 16-byte chunks per thread, all loads issued before stores

template <bool kToTokenMajor>
__global__ void __launch_bounds__(kThreads) permute_rows_kernel(
    const int4* __restrict__ x, int4* __restrict__ y, int N, int chunk_log2, int F, int P,
    const int32_t* __restrict__ mode, bool only_temporal) {
  const int bh = blockIdx.y;
  const bool permute = (mode == nullptr) || (mode[bh] == SVG_MODE_TEMPORAL);
  if (only_temporal && !permute) return;  // this head of y is left as it is
  const long long head_chunks = static_cast<long long>(N) << chunk_log2;
  const int4* xh = x + head_chunks * bh;
  int4* yh = y + head_chunks * bh;
  const long long base = static_cast<long long>(blockIdx.x) * (kThreads * kUnroll) + threadIdx.x;
  const int cmask = (1 << chunk_log2) - 1;

  int4 v[kUnroll];
  long long dst[kUnroll];
#pragma unroll
  for (int i = 0; i < kUnroll; ++i) {
    const long long j = base + i * kThreads;
    dst[i] = j;
    if (j < head_chunks) {
      const int row = static_cast<int>(j >> chunk_log2);
      const int c = static_cast<int>(j) & cmask;
      int src = row;
      if (permute) {
        if (kToTokenMajor) {  // dst m = s F + f  <-  src n = f P + s
          const int s = row / F;
          const int f = row - s * F;
          src = f * P + s;
        } else {  // dst n = f P + s  <-  src m = s F + f
          const int f = row / P;
          const int s = row - f * P;
          src = s * F + f;
        }
      }
      v[i] = __ldcs(xh + ((static_cast<long long>(src) << chunk_log2) | c));
    }
  }
#pragma unroll
  for (int i = 0; i < kUnroll; ++i)
    if (dst[i] < head_chunks) __stcs(yh + dst[i], v[i]);
}

svg_status permute_impl(bool to_token_major, const void* x, void* y, int dtype, int B, int H,
                        int N, int d, int F, int P, const int32_t* mode, void* stream,
                        bool only_temporal = false) {
  clear_error();
  if (only_temporal && mode == nullptr)
    return fail(SVG_ERR_INVALID_ARG, "permute_temporal_heads: mode is required");
  if (x == nullptr || y == nullptr) return fail(SVG_ERR_INVALID_ARG, "permute: null tensor");
  if (dtype != SVG_BF16 && dtype != SVG_FP32)
    return fail(SVG_ERR_INVALID_ARG, "permute: bad dtype %d", dtype);
  if (B <= 0 || H <= 0 || N <= 0 || F <= 0 || P <= 0 || B * H > 65535)
    return fail(SVG_ERR_INVALID_ARG, "permute: bad shape B=%d H=%d N=%d", B, H, N);
  if (static_cast<long long>(F) * P != N)
    return fail(SVG_ERR_INVALID_ARG, "permute: frames*tokens_per_frame (%d*%d) != N (%d)", F, P,
                N);
  if (d != 64 && d != 128) return fail(SVG_ERR_INVALID_ARG, "permute: d=%d not in {64,128}", d);
  if (!aligned16(x) || !aligned16(y))
    return fail(SVG_ERR_INVALID_ARG, "permute: tensors must be 16-byte aligned");
  const long long bytes = static_cast<long long>(B) * H * N * d * elt_bytes(dtype);
  const char* xb = static_cast<const char*>(x);
  const char* yb = static_cast<const char*>(y);
  if (xb < yb + bytes && yb < xb + bytes)
    return fail(SVG_ERR_INVALID_ARG, "permute: x and y overlap (out of place only)");
  const int row_chunks = d * elt_bytes(dtype) / 16;  // 8, 16 or 32
  int chunk_log2 = 0;
  while ((1 << chunk_log2) < row_chunks) ++chunk_log2;
  const long long head_chunks = static_cast<long long>(N) * row_chunks;
  const long long blocks = (head_chunks + kThreads * kUnroll - 1) / (kThreads * kUnroll);
  if (blocks > 0x7fffffffLL) return fail(SVG_ERR_INVALID_ARG, "permute: N too large");
  dim3 grid(static_cast<unsigned>(blocks), B * H);
  auto* xs = static_cast<const int4*>(x);
  auto* ys = static_cast<int4*>(y);
  if (to_token_major)
    permute_rows_kernel<true><<<grid, kThreads, 0, as_stream(stream)>>>(xs, ys, N, chunk_log2, F,
                                                                        P, mode, only_temporal);
  else
    permute_rows_kernel<false><<<grid, kThreads, 0, as_stream(stream)>>>(xs, ys, N, chunk_log2,
                                                                         F, P, mode, false);
  return check_launch("permute");
}

}  // namespace
}  // namespace svg

extern "C" svg_status svg_permute_token_major(const void* x, void* y, int dtype, int B, int H,
                                              int N, int d, int frames, int tokens_per_frame,
                                              const int32_t* mode, void* stream) {
  return svg::permute_impl(true, x, y, dtype, B, H, N, d, frames, tokens_per_frame, mode, stream);
}

extern "C" svg_status svg_permute_frame_major(const void* x, void* y, int dtype, int B, int H,
                                              int N, int d, int frames, int tokens_per_frame,
                                              const int32_t* mode, void* stream) {
  return svg::permute_impl(false, x, y, dtype, B, H, N, d, frames, tokens_per_frame, mode,
                           stream);
}

extern "C" svg_status svg_permute_temporal_heads(const void* x, void* y, int dtype, int B, int H,
                                                 int N, int d, int frames, int tokens_per_frame,
                                                 const int32_t* mode, void* stream) {
  return svg::permute_impl(true, x, y, dtype, B, H, N, d, frames, tokens_per_frame, mode, stream,
                           true);
}
