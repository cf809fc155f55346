// Per-head power-of-two scale that brings V into the fp16 range.
//
// The tcgen05 attention kernel forms P.V with fp16 operands (P in [0, 256]
// keeps 11 significant bits there, against 8 in bf16); V arrives as bf16,
// whose range is far wider.  svg_v_exponents finds for every (b, h) the
// smallest e >= 0 with max |v| * 2^-e <= 65504, the largest finite fp16.
// The attention kernel then converts v * 2^-e (exact: a power of two) and
// multiplies the head's output by 2^e, so any finite bf16 V gives the
// correct result; e = 0 for every head whose values already fit, and then
// nothing changes.
//
// bf16 bits: |v| orders like its 15-bit magnitude field, so the per-head
// maximum is an unsigned max of (bits & 0x7fff).  A finite bf16 value above
// 65504 is at least 2^16, and 1.m * 2^E * 2^-(E - 15) <= 1.9921875 * 2^15 <
// 65504, so e = max(0, E - 15) with E the value's unbiased exponent.  A
// magnitude field of 0x7f80 or more (inf, NaN) gives e = 255: no scale can
// help, and the attention kernel reports SVG_DEVICE_RANGE.
#include "common.cuh"

namespace svg {
namespace {

constexpr int kThreads = 256;
constexpr int kChunksPerThread = 8;  // 16-byte chunks

__global__ void __launch_bounds__(kThreads) v_max_kernel(const uint4* __restrict__ v,
                                                         long long head_chunks,
                                                         int32_t* __restrict__ maxbits) {
  const int bh = blockIdx.y;
  const uint4* vh = v + head_chunks * bh;
  uint32_t m = 0;
  const long long base = static_cast<long long>(blockIdx.x) * kThreads * kChunksPerThread +
                         threadIdx.x;
#pragma unroll
  for (int i = 0; i < kChunksPerThread; ++i) {
    const long long j = base + static_cast<long long>(i) * kThreads;
    if (j < head_chunks) {
      const uint4 c = __ldcs(vh + j);
      for (uint32_t w : {c.x, c.y, c.z, c.w}) m = max(m, max(w & 0x7fffu, (w >> 16) & 0x7fffu));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ uint32_t warp_max[kThreads / 32];
  if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < kThreads / 32; ++w) m = max(m, warp_max[w]);
    atomicMax(reinterpret_cast<unsigned int*>(maxbits + bh), m);
  }
}

__global__ void v_exp_finalize(int32_t* __restrict__ e, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const uint32_t m = static_cast<uint32_t>(e[i]);
  const int E = static_cast<int>(m >> 7) - 127;  // unbiased exponent of the largest |v|
  e[i] = m >= 0x7f80u ? 255 : max(0, E - 15);
}

}  // namespace
}  // namespace svg

using namespace svg;

extern "C" svg_status svg_v_exponents(const void* v, int dtype, int B, int H, int N, int d,
                                      int32_t* exps, void* stream) {
  clear_error();
  if (v == nullptr || exps == nullptr) return fail(SVG_ERR_INVALID_ARG, "v_exponents: null pointer");
  if (dtype != SVG_BF16) return fail(SVG_ERR_UNSUPPORTED, "v_exponents: bf16 only");
  if (B <= 0 || H <= 0 || N <= 0 || B * H > 65535 || (d != 64 && d != 128))
    return fail(SVG_ERR_INVALID_ARG, "v_exponents: bad shape");
  if (!aligned16(v)) return fail(SVG_ERR_INVALID_ARG, "v_exponents: v must be 16-byte aligned");
  cudaStream_t s = as_stream(stream);
  const int bh = B * H;
  if (cudaMemsetAsync(exps, 0, static_cast<size_t>(bh) * sizeof(int32_t), s) != cudaSuccess)
    return fail(SVG_ERR_CUDA, "v_exponents: memset failed");
  const long long head_chunks = static_cast<long long>(N) * d / 8;
  const long long per_block = static_cast<long long>(kThreads) * kChunksPerThread;
  const dim3 grid(static_cast<unsigned>((head_chunks + per_block - 1) / per_block), bh);
  v_max_kernel<<<grid, kThreads, 0, s>>>(static_cast<const uint4*>(v), head_chunks, exps);
  if (svg_status st = check_launch("v_exponents max")) return st;
  v_exp_finalize<<<(bh + 255) / 256, 256, 0, s>>>(exps, bh);
  return check_launch("v_exponents finalize");
}
