// Block energy of dense attention, for calibrated block lists.
//
// CalibAtt article (lpnh.cn/news/568491), section 3.1: for query block r and
// key block c the energy E(r, c) is the attention mass that r's rows put on
// c's keys.  Here E[r, c] = sum_{i in r, j in c} softmax_j(q_i . k_j / sqrt d)
// / |r|, so each row of E sums to 1.
//
// Two passes over every (query tile, key tile) pair of a head:
//   1. lse:    per query row, log2-sum-exp of the scaled scores (workspace);
//   2. energy: per tile pair, the sum of exp2(t_ij - lse_i), reduced into E.
// Both passes are dense QK^T on bf16 tensor cores (mma.sync) with fp32
// accumulation; fp32 inputs use SIMT fp32.  This is an offline step.
#include "common.cuh"
#include "mma_frag.cuh"

namespace svg {
namespace {

constexpr int kQRows = 128;  // query rows per CTA (8 warps x 16)
constexpr int kKeys = 64;    // keys per stage
constexpr int kThreads = 256;
constexpr float kLog2e = 1.4426950408889634f;

template <int D, bool kEnergy>
__global__ void __launch_bounds__(kThreads) energy_pass_bf16(const __nv_bfloat16* __restrict__ q,
                                                             const __nv_bfloat16* __restrict__ k,
                                                             int N, float scale_log2,
                                                             float* __restrict__ lse,
                                                             float* __restrict__ energy) {
  extern __shared__ __align__(128) unsigned char smem[];
  constexpr int TILE = kKeys * D * 2;
  unsigned char* sQ = smem;
  unsigned char* sK = smem + kQRows * D * 2;
  float* eacc = reinterpret_cast<float*>(sK + 2 * TILE);  // [nB] (energy pass)

  const int qt = blockIdx.x, bh = blockIdx.y;
  const int nb = n_tiles(N);
  const long long head = static_cast<long long>(bh) * N * D;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t4 = lane & 3;
  const int row0 = qt * kQRows;
  const int n_rows = min(kQRows, N - row0);

  if (kEnergy)
    for (int c = threadIdx.x; c < nb; c += kThreads) eacc[c] = 0.f;
  load_tile_async<D, kQRows, kThreads>(sQ, q + head, row0, N);
  load_tile_async<D, kKeys, kThreads>(sK, k + head, 0, N);
  cp_async_commit();

  float lrow[2] = {0.f, 0.f};
  float mrow[2] = {-INFINITY, -INFINITY};
  const int r_lo = warp * 16 + g, r_hi = r_lo + 8;
  if (kEnergy) {
    mrow[0] = r_lo < n_rows ? lse[static_cast<long long>(bh) * N + row0 + r_lo] : INFINITY;
    mrow[1] = r_hi < n_rows ? lse[static_cast<long long>(bh) * N + row0 + r_hi] : INFINITY;
  }
  uint32_t qa[D / 16][4];
  const int n_stages = (N + kKeys - 1) / kKeys;
  for (int st = 0; st < n_stages; ++st) {
    if (st + 1 < n_stages) {
      load_tile_async<D, kKeys, kThreads>(sK + ((st + 1) & 1) * TILE, k + head, (st + 1) * kKeys, N);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    if (st == 0) load_a_frags<D>(qa, smem_u32(sQ), warp * 16);
    float s[kKeys / 8][4];
    qk_frags<D, kKeys>(s, qa, smem_u32(sK + (st & 1) * TILE), 0);
    const int key0 = st * kKeys;
    if (!kEnergy) {
      float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int n = 0; n < kKeys / 8; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const bool ok = key0 + 8 * n + 2 * t4 + (e & 1) < N;
          s[n][e] = ok ? s[n][e] * scale_log2 : -INFINITY;
          mx[e >> 1] = fmaxf(mx[e >> 1], s[n][e]);
        }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
        mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
        const float mn = fmaxf(mrow[h], mx[h]);
        lrow[h] *= fast_exp2(mrow[h] - mn);
        mrow[h] = mn;
#pragma unroll
        for (int n = 0; n < kKeys / 8; ++n)
          lrow[h] += fast_exp2(s[n][2 * h] - mn) + fast_exp2(s[n][2 * h + 1] - mn);
      }
    } else {
      float part = 0.f;
#pragma unroll
      for (int n = 0; n < kKeys / 8; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const bool ok = key0 + 8 * n + 2 * t4 + (e & 1) < N;
          if (ok) part += fast_exp2(s[n][e] * scale_log2 - mrow[e >> 1]);
        }
#pragma unroll
      for (int o2 = 16; o2 > 0; o2 >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o2);
      if (lane == 0) atomicAdd(&eacc[key0 / SVG_TILE], part);
    }
    __syncthreads();
  }
  if (!kEnergy) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      lrow[h] += __shfl_xor_sync(0xffffffffu, lrow[h], 1);
      lrow[h] += __shfl_xor_sync(0xffffffffu, lrow[h], 2);
      const int r = h ? r_hi : r_lo;
      if (t4 == 0 && r < n_rows)
        lse[static_cast<long long>(bh) * N + row0 + r] = mrow[h] + __log2f(lrow[h]);
    }
  } else {
    float* out = energy + (static_cast<long long>(bh) * nb + qt) * nb;
    const float inv = 1.f / static_cast<float>(n_rows);
    for (int c = threadIdx.x; c < nb; c += kThreads) out[c] = eacc[c] * inv;
  }
}

// fp32 SIMT: one thread per query row.
template <int D, bool kEnergy>
__global__ void __launch_bounds__(128) energy_pass_fp32(const float* __restrict__ q,
                                                        const float* __restrict__ k, int N,
                                                        float scale_log2, float* __restrict__ lse,
                                                        float* __restrict__ energy) {
  extern __shared__ float eacc[];  // [nB]
  const int qt = blockIdx.x, bh = blockIdx.y;
  const int nb = n_tiles(N);
  const long long head = static_cast<long long>(bh) * N * D;
  const int row = qt * SVG_TILE + threadIdx.x;
  const bool valid = threadIdx.x < SVG_TILE && row < N;
  if (kEnergy)
    for (int c = threadIdx.x; c < nb; c += blockDim.x) eacc[c] = 0.f;
  __syncthreads();
  float m = -INFINITY, l = 0.f;
  const float l2 = (kEnergy && valid) ? lse[static_cast<long long>(bh) * N + row] : 0.f;
  for (int c = 0; c < nb; ++c) {
    float part = 0.f;
    if (valid) {
      for (int j = c * SVG_TILE; j < min(N, (c + 1) * SVG_TILE); ++j) {
        float dot = 0.f;
        for (int e = 0; e < D; ++e)
          dot = fmaf(q[head + static_cast<long long>(row) * D + e], k[head + static_cast<long long>(j) * D + e], dot);
        const float t = dot * scale_log2;
        if (kEnergy) {
          part += exp2f(t - l2);
        } else {
          const float mn = fmaxf(m, t);
          l = l * exp2f(m - mn) + exp2f(t - mn);
          m = mn;
        }
      }
    }
    if (kEnergy) {
#pragma unroll
      for (int o2 = 16; o2 > 0; o2 >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o2);
      if ((threadIdx.x & 31) == 0) atomicAdd(&eacc[c], part);
    }
  }
  if (!kEnergy) {
    if (valid) lse[static_cast<long long>(bh) * N + row] = m + log2f(l);
  } else {
    __syncthreads();
    const int n_rows = min(SVG_TILE, N - qt * SVG_TILE);
    float* out = energy + (static_cast<long long>(bh) * nb + qt) * nb;
    for (int c = threadIdx.x; c < nb; c += blockDim.x) out[c] = eacc[c] / static_cast<float>(n_rows);
  }
}

template <int D>
svg_status launch_energy(const void* q, const void* k, int dtype, int B, int H, int N,
                         float* energy, float* lse, cudaStream_t s) {
  const int nb = n_tiles(N);
  const float scale_log2 = kLog2e / sqrtf(static_cast<float>(D));
  dim3 grid(nb, B * H);
  if (dtype == SVG_BF16) {
    const size_t base = static_cast<size_t>(kQRows) * D * 2 + 2 * static_cast<size_t>(kKeys) * D * 2;
    const size_t smem_e = base + static_cast<size_t>(nb) * 4;
    if (smem_e > 227 * 1024) return fail(SVG_ERR_UNSUPPORTED, "block_energy: N too large");
    auto* qb = static_cast<const __nv_bfloat16*>(q);
    auto* kb = static_cast<const __nv_bfloat16*>(k);
    if (cudaFuncSetAttribute(energy_pass_bf16<D, false>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(base)) != cudaSuccess ||
        cudaFuncSetAttribute(energy_pass_bf16<D, true>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem_e)) != cudaSuccess)
      return fail(SVG_ERR_CUDA, "block_energy: cannot reserve shared memory");
    energy_pass_bf16<D, false><<<grid, kThreads, base, s>>>(qb, kb, N, scale_log2, lse, energy);
    if (svg_status st = check_launch("block_energy lse")) return st;
    energy_pass_bf16<D, true><<<grid, kThreads, smem_e, s>>>(qb, kb, N, scale_log2, lse, energy);
  } else {
    const size_t smem_e = static_cast<size_t>(nb) * 4;
    if (smem_e > 48 * 1024) return fail(SVG_ERR_UNSUPPORTED, "block_energy: N too large for fp32");
    auto* qf = static_cast<const float*>(q);
    auto* kf = static_cast<const float*>(k);
    energy_pass_fp32<D, false><<<grid, 128, 0, s>>>(qf, kf, N, scale_log2, lse, energy);
    if (svg_status st = check_launch("block_energy lse")) return st;
    energy_pass_fp32<D, true><<<grid, 128, smem_e, s>>>(qf, kf, N, scale_log2, lse, energy);
  }
  return check_launch("block_energy");
}

}  // namespace
}  // namespace svg

using namespace svg;

extern "C" size_t svg_block_energy_workspace_size(int B, int H, int N) {
  if (B <= 0 || H <= 0 || N <= 0) return 0;
  return (static_cast<size_t>(B) * H * N * sizeof(float) + 255) / 256 * 256;
}

extern "C" svg_status svg_block_energy(const void* q, const void* k, int dtype, int B, int H, int N,
                                       int d, float* energy, void* workspace,
                                       size_t workspace_bytes, void* stream) {
  clear_error();
  if (q == nullptr || k == nullptr || energy == nullptr)
    return fail(SVG_ERR_INVALID_ARG, "block_energy: null pointer");
  if (dtype != SVG_BF16 && dtype != SVG_FP32)
    return fail(SVG_ERR_INVALID_ARG, "block_energy: bad dtype %d", dtype);
  if (B <= 0 || H <= 0 || N <= 0 || B * H > 65535)
    return fail(SVG_ERR_INVALID_ARG, "block_energy: bad shape");
  if (d != 64 && d != 128) return fail(SVG_ERR_INVALID_ARG, "block_energy: d=%d not in {64,128}", d);
  if (!aligned16(q) || !aligned16(k))
    return fail(SVG_ERR_INVALID_ARG, "block_energy: tensors must be 16-byte aligned");
  if (workspace == nullptr || !aligned256(workspace) ||
      workspace_bytes < svg_block_energy_workspace_size(B, H, N))
    return fail(SVG_ERR_INVALID_ARG, "block_energy: workspace too small or not 256-byte aligned");
  auto* lse = static_cast<float*>(workspace);
  cudaStream_t s = as_stream(stream);
  if (d == 64) return launch_energy<64>(q, k, dtype, B, H, N, energy, lse, s);
  return launch_energy<128>(q, k, dtype, B, H, N, energy, lse, s);
}
