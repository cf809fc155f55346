// QK-Norm + rotary position embedding of q and k, with token-major copies.
//
// Sparse VideoGen article (m.jxzklqfsx.com/article/815093.html), section
// "Layout Transformation + Kernel 加速": beside the attention kernels the
// method ships its own QK-Norm and RoPE kernels.  This kernel does both for
// q and k in one pass and, optionally, writes the token-major copy
// (m = s F + f) of every head in the same pass, so that the layer's
// reordering of q and k costs no extra read.
//
//   x_hat = x / sqrt(mean_c x_c^2 + eps) * gamma          (QK-Norm, per row)
//   (a, b) = (x_hat[2i], x_hat[2i+1]) -> (a cos - b sin, a sin + b cos)
//                                                         (RoPE, per pair)
//
// HBM-bound: per row it reads q and k once and writes two or four rows.
// Thread layout: 16-byte chunks, CPR of them per row, kThreads / CPR rows per
// pass.  A work unit is one window of those rows times a group of heads; a
// thread keeps the same (row of the window, chunk) for every head of the
// unit, so its weights and its cos / sin values stay in registers and each
// head costs it one 16-byte load of q and of k.
#include "common.cuh"

namespace svg {
namespace {

constexpr int kThreads = 256;
constexpr int kHeadsPerUnit = 4;  // heads sharing one load of the cos / sin window
constexpr int kHeadUnroll = 4;    // heads whose loads are in flight together

template <typename T>
struct Elems;
template <>
struct Elems<__nv_bfloat16> {
  static constexpr int kPerChunk = 8;
};
template <>
struct Elems<float> {
  static constexpr int kPerChunk = 4;
};

template <typename T>
__device__ __forceinline__ void chunk_to_float(const int4& v, float* x);
template <>
__device__ __forceinline__ void chunk_to_float<__nv_bfloat16>(const int4& v, float* x) {
  const uint32_t w[4] = {static_cast<uint32_t>(v.x), static_cast<uint32_t>(v.y),
                         static_cast<uint32_t>(v.z), static_cast<uint32_t>(v.w)};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = __uint_as_float(w[i] << 16);
    x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}
template <>
__device__ __forceinline__ void chunk_to_float<float>(const int4& v, float* x) {
  x[0] = __int_as_float(v.x);
  x[1] = __int_as_float(v.y);
  x[2] = __int_as_float(v.z);
  x[3] = __int_as_float(v.w);
}

template <typename T>
__device__ __forceinline__ int4 float_to_chunk(const float* x);
template <>
__device__ __forceinline__ int4 float_to_chunk<__nv_bfloat16>(const float* x) {
  return make_int4(static_cast<int>(pack_bf16x2(x[0], x[1])),
                   static_cast<int>(pack_bf16x2(x[2], x[3])),
                   static_cast<int>(pack_bf16x2(x[4], x[5])),
                   static_cast<int>(pack_bf16x2(x[6], x[7])));
}
template <>
__device__ __forceinline__ int4 float_to_chunk<float>(const float* x) {
  return make_int4(__float_as_int(x[0]), __float_as_int(x[1]), __float_as_int(x[2]),
                   __float_as_int(x[3]));
}

// HP consecutive table values (16 or 8 bytes, aligned: rows are d/2 floats).
template <int HP>
__device__ __forceinline__ void load_pairs(const float* p, float* out);
template <>
__device__ __forceinline__ void load_pairs<4>(const float* p, float* out) {
  const float4 v = __ldg(reinterpret_cast<const float4*>(p));
  out[0] = v.x;
  out[1] = v.y;
  out[2] = v.z;
  out[3] = v.w;
}
template <>
__device__ __forceinline__ void load_pairs<2>(const float* p, float* out) {
  const float2 v = __ldg(reinterpret_cast<const float2*>(p));
  out[0] = v.x;
  out[1] = v.y;
}

struct QkArgs {
  const int4* q;
  const int4* k;
  int4* q_out;
  int4* k_out;
  int4* q_tm;  // token-major copies, or null
  int4* k_tm;
  const float* gamma_q;  // [d] or null (weight 1)
  const float* gamma_k;
  const float* cos;  // [N][d/2]
  const float* sin;
  float eps;
  int BH, N, F, P;
  bool norm, rope;
};

// One 16-byte chunk of one row: normalise with the row's sum of squares
// (reduced over the CPR lanes that hold the row) and rotate its pairs.
template <typename T, int D>
__device__ __forceinline__ int4 transform(const int4 v, const float* g, const float* cs,
                                          const float* sn, const QkArgs& a) {
  constexpr int E = Elems<T>::kPerChunk, CPR = D / E;
  float x[E];
  chunk_to_float<T>(v, x);
  if (a.norm) {
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) ss = fmaf(x[e], x[e], ss);
#pragma unroll
    for (int o = CPR / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float rs = rsqrtf(ss * (1.0f / D) + a.eps);
#pragma unroll
    for (int e = 0; e < E; ++e) x[e] = x[e] * rs * g[e];
  }
  if (a.rope) {
#pragma unroll
    for (int i = 0; i < E / 2; ++i) {
      const float p = x[2 * i], q = x[2 * i + 1];
      x[2 * i] = p * cs[i] - q * sn[i];
      x[2 * i + 1] = p * sn[i] + q * cs[i];
    }
  }
  return float_to_chunk<T>(x);
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads, 3) qk_norm_rope_kernel(const QkArgs a) {
  constexpr int E = Elems<T>::kPerChunk, CPR = D / E, RP = kThreads / CPR, HP = E / 2;
  const int c = threadIdx.x % CPR, r = threadIdx.x / CPR;
  float gq[E], gk[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    gq[e] = a.gamma_q != nullptr ? a.gamma_q[c * E + e] : 1.f;
    gk[e] = a.gamma_k != nullptr ? a.gamma_k[c * E + e] : 1.f;
  }
  const int N = a.N;
  const int n_windows = (N + RP - 1) / RP;
  const int n_groups = (a.BH + kHeadsPerUnit - 1) / kHeadsPerUnit;
  const long long units = static_cast<long long>(n_windows) * n_groups;
  for (long long u = blockIdx.x; u < units; u += gridDim.x) {
    const int g = static_cast<int>(u / n_windows);
    const int n = static_cast<int>(u - static_cast<long long>(g) * n_windows) * RP + r;
    const bool valid = n < N;
    float cs[HP], sn[HP];
#pragma unroll
    for (int i = 0; i < HP; ++i) {
      cs[i] = 1.f;
      sn[i] = 0.f;
    }
    if (a.rope && valid) {
      const long long t = static_cast<long long>(n) * (D / 2) + c * HP;
      load_pairs<HP>(a.cos + t, cs);
      load_pairs<HP>(a.sin + t, sn);
    }
    // token-major row of token n = f P + s is m = s F + f
    const int m = (a.q_tm != nullptr && valid) ? (n % a.P) * a.F + n / a.P : 0;
    const int bh0 = g * kHeadsPerUnit;
    const int bh1 = min(a.BH, bh0 + kHeadsPerUnit);
    for (int bh = bh0; bh < bh1; bh += kHeadUnroll) {
      int4 vq[kHeadUnroll], vk[kHeadUnroll];
#pragma unroll
      for (int i = 0; i < kHeadUnroll; ++i) {
        vq[i] = vk[i] = make_int4(0, 0, 0, 0);
        if (valid && bh + i < bh1) {
          const long long off = (static_cast<long long>(bh + i) * N + n) * CPR + c;
          vq[i] = __ldcs(a.q + off);
          vk[i] = __ldcs(a.k + off);
        }
      }
#pragma unroll
      for (int i = 0; i < kHeadUnroll; ++i) {
        // every lane takes part in the row reductions; only stores are guarded
        const int4 yq = transform<T, D>(vq[i], gq, cs, sn, a);
        const int4 yk = transform<T, D>(vk[i], gk, cs, sn, a);
        if (valid && bh + i < bh1) {
          const long long head = static_cast<long long>(bh + i) * N;
          a.q_out[(head + n) * CPR + c] = yq;
          a.k_out[(head + n) * CPR + c] = yk;
          if (a.q_tm != nullptr) {
            a.q_tm[(head + m) * CPR + c] = yq;
            a.k_tm[(head + m) * CPR + c] = yk;
          }
        }
      }
    }
  }
}

bool overlaps(const void* a, const void* b, long long bytes) {
  const char* x = static_cast<const char*>(a);
  const char* y = static_cast<const char*>(b);
  return x < y + bytes && y < x + bytes;
}

template <typename T, int D>
svg_status launch(const QkArgs& a, cudaStream_t s) {
  constexpr int E = Elems<T>::kPerChunk, RP = kThreads / (D / E);
  const long long units = static_cast<long long>((a.N + RP - 1) / RP) *
                          ((a.BH + kHeadsPerUnit - 1) / kHeadsPerUnit);
  // one wave of resident CTAs walks the units (occupancy cached per device)
  static int per_sm_cache[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  int per_sm = dev >= 0 && dev < 64 ? per_sm_cache[dev] : 0;
  if (per_sm == 0) {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, qk_norm_rope_kernel<T, D>,
                                                      kThreads, 0) != cudaSuccess ||
        per_sm < 1) {
      (void)cudaGetLastError();
      per_sm = 1;
    }
    if (dev >= 0 && dev < 64) per_sm_cache[dev] = per_sm;
  }
  const long long cap = static_cast<long long>(sm_count()) * per_sm;
  const int grid = static_cast<int>(units < cap ? units : cap);
  qk_norm_rope_kernel<T, D><<<grid, kThreads, 0, s>>>(a);
  return check_launch("qk_norm_rope");
}

}  // namespace
}  // namespace svg

using namespace svg;

extern "C" svg_status svg_qk_norm_rope(const void* q, const void* k, void* q_out, void* k_out,
                                       void* q_tm_out, void* k_tm_out, int dtype, int B, int H,
                                       int N, int d, int frames, int tokens_per_frame, int ops,
                                       const float* gamma_q, const float* gamma_k, float eps,
                                       const float* rope_cos, const float* rope_sin,
                                       void* stream) {
  clear_error();
  if (q == nullptr || k == nullptr || q_out == nullptr || k_out == nullptr)
    return fail(SVG_ERR_INVALID_ARG, "qk_norm_rope: null tensor");
  if (dtype != SVG_BF16 && dtype != SVG_FP32)
    return fail(SVG_ERR_INVALID_ARG, "qk_norm_rope: bad dtype %d", dtype);
  if (B <= 0 || H <= 0 || N <= 0 || static_cast<long long>(B) * H > 0x7fffffffLL)
    return fail(SVG_ERR_INVALID_ARG, "qk_norm_rope: bad shape B=%d H=%d N=%d", B, H, N);
  if (d != 64 && d != 128)
    return fail(SVG_ERR_INVALID_ARG, "qk_norm_rope: d=%d not in {64,128}", d);
  if ((ops & ~(SVG_QK_NORM | SVG_QK_ROPE)) != 0)
    return fail(SVG_ERR_INVALID_ARG, "qk_norm_rope: bad ops 0x%x", ops);
  const bool norm = (ops & SVG_QK_NORM) != 0, rope = (ops & SVG_QK_ROPE) != 0;
  if (norm && !(eps >= 0.f && eps < 3.0e38f))
    return fail(SVG_ERR_INVALID_ARG, "qk_norm_rope: eps must be finite and >= 0");
  if (rope && (rope_cos == nullptr || rope_sin == nullptr))
    return fail(SVG_ERR_INVALID_ARG, "qk_norm_rope: RoPE needs cos and sin tables");
  if ((q_tm_out == nullptr) != (k_tm_out == nullptr))
    return fail(SVG_ERR_INVALID_ARG, "qk_norm_rope: give both token-major outputs or neither");
  const bool tm = q_tm_out != nullptr;
  if (tm && (frames <= 0 || tokens_per_frame <= 0 ||
             static_cast<long long>(frames) * tokens_per_frame != N))
    return fail(SVG_ERR_INVALID_ARG, "qk_norm_rope: frames*tokens_per_frame (%d*%d) != N (%d)",
                frames, tokens_per_frame, N);
  const void* ptrs[] = {q, k, q_out, k_out, q_tm_out, k_tm_out, gamma_q, gamma_k, rope_cos,
                        rope_sin};
  for (const void* p : ptrs)
    if (p != nullptr && !aligned16(p))
      return fail(SVG_ERR_INVALID_ARG, "qk_norm_rope: pointers must be 16-byte aligned");
  const long long bytes = static_cast<long long>(B) * H * N * d * elt_bytes(dtype);
  // q_out may be q itself (in place) and k_out k itself; nothing else overlaps
  if ((q_out != q && overlaps(q_out, q, bytes)) || overlaps(q_out, k, bytes) ||
      (k_out != k && overlaps(k_out, k, bytes)) || overlaps(k_out, q, bytes) ||
      overlaps(q_out, k_out, bytes))
    return fail(SVG_ERR_INVALID_ARG, "qk_norm_rope: outputs overlap the inputs or each other");
  if (tm) {
    const void* others[] = {q, k, q_out, k_out};
    for (const void* p : others)
      if (overlaps(q_tm_out, p, bytes) || overlaps(k_tm_out, p, bytes))
        return fail(SVG_ERR_INVALID_ARG, "qk_norm_rope: token-major outputs overlap a tensor");
    if (overlaps(q_tm_out, k_tm_out, bytes))
      return fail(SVG_ERR_INVALID_ARG, "qk_norm_rope: token-major outputs overlap each other");
  }
  QkArgs a;
  a.q = static_cast<const int4*>(q);
  a.k = static_cast<const int4*>(k);
  a.q_out = static_cast<int4*>(q_out);
  a.k_out = static_cast<int4*>(k_out);
  a.q_tm = static_cast<int4*>(q_tm_out);
  a.k_tm = static_cast<int4*>(k_tm_out);
  a.gamma_q = norm ? gamma_q : nullptr;
  a.gamma_k = norm ? gamma_k : nullptr;
  a.cos = rope_cos;
  a.sin = rope_sin;
  a.eps = eps;
  a.BH = B * H;
  a.N = N;
  a.F = tm ? frames : 1;
  a.P = tm ? tokens_per_frame : N;
  a.norm = norm;
  a.rope = rope;
  cudaStream_t s = as_stream(stream);
  if (dtype == SVG_BF16)
    return d == 64 ? launch<__nv_bfloat16, 64>(a, s) : launch<__nv_bfloat16, 128>(a, s);
  return d == 64 ? launch<float, 64>(a, s) : launch<float, 128>(a, s);
}
