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
// Both passes are dense Q K^T; bf16 inputs on the tcgen05 tensor core with
// the scores in TMEM, fp32 inputs in SIMT fp32.  This is an offline step.
#include "common.cuh"
#include "sm100.cuh"

namespace svg {
namespace {

constexpr float kLog2e = 1.4426950408889634f;

// tcgen05 passes (bf16): persistent, one CTA per SM, looping over units
// (query tile r, head).  Warp 8 loads the unit's Q tile and streams every K
// tile of the head through a ring (TMA); warp 9 issues S_j = Q K_j^T
// (tcgen05.mma, M = 128, N = 128) into one of two TMEM score buffers; warps
// 0-7 read the scores, warp w taking TMEM lanes 32 (w & 3) .. + 31 (query
// rows) and key columns 64 (w >> 2) .. + 63 of every tile:
//   lse pass:    online max and sum of exp2 per row and column half, the two
//                halves merged through shared memory at the unit's end;
//   energy pass: per tile, the sum of exp2(t - lse) over the warp's rows and
//                columns, added into the unit's row of E in shared memory
//                (one shared atomic per warp and tile), written out at the
//                unit's end.
// Every wait is bounded; a CTA that gives up writes NaN (lse pass: the rows'
// lse, energy pass: the unit's energies) and drains.

constexpr int kEnThreads = 320;  // 10 warps
constexpr uint32_t kEnSpin = 1u << 22;
constexpr uint32_t kEnDrain = 1u << 20;

template <int D>
struct EnCfg {
  static constexpr int kTile = 128 * D * 2;         // a 128-row Q / K tile
  static constexpr int kBox = 16384;                // 128 rows x 128 bytes
  static constexpr int kBoxes = D / 64;
  static constexpr int kStages = D == 64 ? 8 : 4;   // K ring entries
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kTile;
  static constexpr int kOffBar = kOffK + kStages * kTile;
  // q_full, q_empty, k_full[S], k_empty[S], s_full[2], s_free[2], xfull[4],
  // xdone[4], added, cleared, drain
  static constexpr int kBars = 2 + 2 * kStages + 2 + 2 + 4 + 4 + 3;
  static constexpr int kOffX = kOffBar + kBars * 8 + 16;  // float [4][32][2]
  static constexpr int kOffE = kOffX + 1024;              // float eacc[nB]
  static constexpr uint32_t kIdescQK = sm100::idesc_bf16(128, 128, false);
  static size_t smem(int nb) { return kOffE + static_cast<size_t>(nb) * 4 + 1024; }
};

__device__ __forceinline__ bool en_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  const uint32_t addr = smem_u32(bar);
  for (uint32_t i = 0; i < kEnSpin; ++i) {
    if (sm100::mbar_try_wait(addr, parity)) return true;
    if ((i & 255u) == 255u && *abort_flag) return false;
  }
  *abort_flag = 1;
  return false;
}
// the same, taken by a whole warp: every lane leaves with the same answer
__device__ __forceinline__ bool en_wait_warp(uint64_t* bar, uint32_t parity,
                                             volatile int* abort_flag) {
  return __all_sync(0xffffffffu, en_wait(bar, parity, abort_flag)) != 0;
}
__device__ __forceinline__ void en_drain(uint64_t* bar, uint32_t parity) {
  const uint32_t addr = smem_u32(bar);
  for (uint32_t i = 0; i < kEnDrain; ++i)
    if (sm100::mbar_try_wait(addr, parity)) return;
}

template <int D, bool kEnergy>
__global__ void __launch_bounds__(kEnThreads, 1) energy_pass_tc(
    const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk, int N,
    int n_units, float scale_log2, float* __restrict__ lse, float* __restrict__ energy) {
  using C = EnCfg<D>;
  using namespace sm100;
  constexpr int ST = C::kStages;
  const int nb = n_tiles(N);
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* q_full = bars;
  uint64_t* q_empty = bars + 1;
  uint64_t* k_full = bars + 2;
  uint64_t* k_empty = k_full + ST;
  uint64_t* s_full = k_empty + ST;
  uint64_t* s_free = s_full + 2;
  uint64_t* xfull = s_free + 2;   // [4] lse pass: half 1 has posted its (max, sum)
  uint64_t* xdone = xfull + 4;    // [4] lse pass: half 0 has read them
  uint64_t* added = xdone + 4;    // energy pass: the 8 warps have added the unit's tiles
  uint64_t* cleared = added + 1;  // energy pass: the unit's row of E is written and zeroed
  uint64_t* drain = cleared + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* eacc = reinterpret_cast<float*>(smem + C::kOffE);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (kEnergy)
    for (int c = threadIdx.x; c < nb; c += kEnThreads) eacc[c] = 0.f;
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < ST; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_free[b], 8);
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(&xfull[i], 1);
      mbar_init(&xdone[i], 1);
    }
    mbar_init(added, 8);
    mbar_init(cleared, 8);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 8) {
    // ------------------------------------------------------------------ loader
    if (lane == 0) {
      prefetch_tmap(&mq);
      prefetch_tmap(&mk);
      uint32_t gk = 0, nu = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        const int bh = u / nb, qt = u - bh * nb;
        if (!(ok = en_wait(q_empty, (nu & 1) ^ 1, abort_flag))) break;
        mbar_arrive_expect_tx(q_full, C::kTile);
        for (int bx = 0; bx < C::kBoxes; ++bx)
          tma_load_3d(smem + C::kOffQ + bx * C::kBox, &mq, q_full, 64 * bx, qt * 128, bh);
        ++nu;
        for (int j = 0; j < nb; ++j, ++gk) {
          const uint32_t st = gk % ST;
          if (!(ok = en_wait(&k_empty[st], ((gk / ST) & 1) ^ 1, abort_flag))) break;
          mbar_arrive_expect_tx(&k_full[st], C::kTile);
          for (int bx = 0; bx < C::kBoxes; ++bx)
            tma_load_3d(smem + C::kOffK + st * C::kTile + bx * C::kBox, &mk, &k_full[st], 64 * bx,
                        j * 128, bh);
        }
      }
      if (!ok) {  // copies in flight land before the CTA can exit
        for (uint32_t l = gk > ST ? gk - ST : 0; l < gk; ++l) en_drain(&k_full[l % ST], (l / ST) & 1);
        if (nu > 0) en_drain(q_full, (nu - 1) & 1);
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint64_t dq = sdesc_sw128(smem_u32(smem + C::kOffQ), 16, 1024);
      const uint64_t dk = sdesc_sw128(smem_u32(smem + C::kOffK), 16, 1024);
      uint32_t gk = 0, nu = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        if (!(ok = en_wait(q_full, nu & 1, abort_flag))) break;
        tc_fence_after();
        for (int j = 0; j < nb; ++j, ++gk) {
          const uint32_t st = gk % ST, b = gk & 1;
          if (!(ok = en_wait(&k_full[st], (gk / ST) & 1, abort_flag))) break;
          // the softmax warps have read S_b (two tiles back)
          if (!(ok = en_wait(&s_free[b], ((gk >> 1) & 1) ^ 1, abort_flag))) break;
          tc_fence_after();
          const uint64_t k0 = dk + ((st * C::kTile) >> 4);
          if constexpr (D == 64)
            mma_ss_k64(tmem + 128 * b, dq, k0, C::kIdescQK);
          else
            mma_ss_k128(tmem + 128 * b, dq, k0, C::kIdescQK, C::kBox >> 4);
          tc_commit(&s_full[b]);
          tc_commit(&k_empty[st]);
          if (j == nb - 1) tc_commit(q_empty);  // the unit's last Q K^T
        }
        ++nu;
      }
      tc_commit(drain);  // every MMA completes before TMEM is released
      en_drain(drain, 0);
    }
  } else {
    // ------------------------------------------------------------------ scores
    const int quarter = warp & 3, half = warp >> 2;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    volatile float* xv = reinterpret_cast<volatile float*>(smem + C::kOffX) + (quarter * 32 + lane) * 2;
    uint32_t gk = 0, xph = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
      const int bh = u / nb, qt = u - bh * nb;
      const int n = qt * 128 + row;  // query row
      const bool valid = n < N;
      // energy pass: exp2(t - lse) of a valid row; -inf offset (weights 0) else
      const float neg = kEnergy ? (valid ? -lse[static_cast<long long>(bh) * N + n] : -INFINITY) : 0.f;
      float m = -INFINITY, l = 0.f;
      for (int j = 0; j < nb; ++j, ++gk) {
        const uint32_t b = gk & 1;
        if (!(ok = en_wait_warp(&s_full[b], (gk >> 1) & 1, abort_flag))) break;
        tc_fence_after();
        float s[64];
        {
          uint32_t rr[2][32];
          tmem_ld32(tmem + lane_off + 128 * b + 64 * half, rr[0]);
          tmem_ld32(tmem + lane_off + 128 * b + 64 * half + 32, rr[1]);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            reg_fence32(rr[c]);
#pragma unroll
            for (int i = 0; i < 32; ++i) s[32 * c + i] = __uint_as_float(rr[c][i]);
          }
        }
        // S_b is in registers: the next Q K^T may overwrite it
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_free[b]);
        const int vc = N - (j * 128 + 64 * half);  // valid key columns of this half
        if (vc < 64) {
#pragma unroll
          for (int i = 0; i < 64; ++i) s[i] = i < vc ? s[i] : -INFINITY;
        }
        if constexpr (!kEnergy) {
          float m4[4] = {s[0], s[1], s[2], s[3]};
#pragma unroll
          for (int i = 4; i < 60; i += 8)
#pragma unroll
            for (int c = 0; c < 4; ++c) m4[c] = sm100::max3(m4[c], s[i + c], s[i + 4 + c]);
          const float mx = sm100::max3(sm100::max3(m4[0], s[60], s[61]),
                                       sm100::max3(m4[1], s[62], s[63]), fmaxf(m4[2], m4[3])) *
                           scale_log2;
          if (mx > m) {
            if (m != -INFINITY) l *= exp2f(m - mx);
            m = mx;
          }
          const float o = m == -INFINITY ? -INFINITY : -m;
          float l0 = 0.f, l1 = 0.f;
#pragma unroll
          for (int i = 0; i < 64; i += 2) {
            float t0, t1;
            sm100::fma2(t0, t1, s[i], s[i + 1], scale_log2, scale_log2, o, o);
            l0 += fast_exp2(t0);
            l1 += fast_exp2(t1);
          }
          l += l0 + l1;
        } else {
          float p0 = 0.f, p1 = 0.f;
#pragma unroll
          for (int i = 0; i < 64; i += 2) {
            float t0, t1;
            sm100::fma2(t0, t1, s[i], s[i + 1], scale_log2, scale_log2, neg, neg);
            p0 += fast_exp2(t0);
            p1 += fast_exp2(t1);
          }
          float part = p0 + p1;
#pragma unroll
          for (int o2 = 16; o2 > 0; o2 >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o2);
          if (lane == 0) atomicAdd(&eacc[j], part);
        }
      }
      if (!ok) break;
      if constexpr (!kEnergy) {
        // merge the two column halves of each row: lse = M + log2 L
        if (half == 1) {
          xv[0] = m;
          xv[1] = l;
          __syncwarp();
          if (lane == 0) mbar_arrive(&xfull[quarter]);
          if (!(ok = en_wait_warp(&xdone[quarter], xph & 1, abort_flag))) break;
        } else {
          if (!(ok = en_wait_warp(&xfull[quarter], xph & 1, abort_flag))) break;
          const float m1 = xv[0], l1 = xv[1];
          const float mm = fmaxf(m, m1);
          const float ll = (m == -INFINITY ? 0.f : l * exp2f(m - mm)) +
                           (m1 == -INFINITY ? 0.f : l1 * exp2f(m1 - mm));
          if (valid) lse[static_cast<long long>(bh) * N + n] = mm + __log2f(ll);
          __syncwarp();
          if (lane == 0) mbar_arrive(&xdone[quarter]);
        }
      } else {
        // every warp has added the unit's tiles: write the row of E, zero it
        __syncwarp();
        if (lane == 0) mbar_arrive(added);
        if (!(ok = en_wait_warp(added, xph & 1, abort_flag))) break;
        const float inv = 1.f / static_cast<float>(min(128, N - qt * 128));
        float* out = energy + (static_cast<long long>(bh) * nb + qt) * nb;
        for (int c = threadIdx.x; c < nb; c += 256) {
          out[c] = eacc[c] * inv;
          eacc[c] = 0.f;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(cleared);
        if (!(ok = en_wait_warp(cleared, xph & 1, abort_flag))) break;
      }
      ++xph;
    }
    if (!ok) {
      // a wait gave up: this CTA's results are not to be trusted
      for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
        const int bh = u / nb, qt = u - bh * nb;
        if (!kEnergy) {
          const int n = qt * 128 + row;
          if (half == 0 && n < N) lse[static_cast<long long>(bh) * N + n] = __int_as_float(0x7fc00000);
        } else {
          float* out = energy + (static_cast<long long>(bh) * nb + qt) * nb;
          for (int c = threadIdx.x; c < nb; c += 256) out[c] = __int_as_float(0x7fc00000);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 9) tmem_dealloc(tmem, 256);
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
  if (dtype == SVG_BF16) {
    using C = EnCfg<D>;
    const size_t smem = C::smem(nb);
    if (smem > 227 * 1024) return fail(SVG_ERR_UNSUPPORTED, "block_energy: N too large");
    CUtensorMap mq, mk;
    if (!make_tma_map_3d(&mq, q, B * H, N, D) || !make_tma_map_3d(&mk, k, B * H, N, D))
      return fail(SVG_ERR_CUDA, "block_energy: cannot encode TMA descriptors");
    if (cudaFuncSetAttribute(energy_pass_tc<D, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess ||
        cudaFuncSetAttribute(energy_pass_tc<D, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return fail(SVG_ERR_CUDA, "block_energy: cannot reserve shared memory");
    const long long units = static_cast<long long>(B) * H * nb;
    if (units > 0x7fffffffLL) return fail(SVG_ERR_UNSUPPORTED, "block_energy: too many tiles");
    const int grid = static_cast<int>(units < sm_count() ? units : sm_count());
    energy_pass_tc<D, false><<<grid, kEnThreads, smem, s>>>(mq, mk, N, static_cast<int>(units),
                                                            scale_log2, lse, energy);
    if (svg_status st = check_launch("block_energy lse")) return st;
    energy_pass_tc<D, true><<<grid, kEnThreads, smem, s>>>(mq, mk, N, static_cast<int>(units),
                                                           scale_log2, lse, energy);
  } else {
    const size_t smem_e = static_cast<size_t>(nb) * 4;
    if (smem_e > 48 * 1024) return fail(SVG_ERR_UNSUPPORTED, "block_energy: N too large for fp32");
    auto* qf = static_cast<const float*>(q);
    auto* kf = static_cast<const float*>(k);
    const dim3 grid(nb, B * H);
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
