// Block-sparse attention on the B200 tensor core (tcgen05 + TMEM + TMA).
//
// Video-diffusion acceleration survey (wmrh.cn/news/48564), section 2.1:
// o = softmax(Q K^T / sqrt(d_k)) V; section 5.3: tiled on chip with an online
// softmax.  CalibAtt article (lpnh.cn/news/568491), sections 2.2 and 3.3:
// keep/skip decisions on 128 x 128 tiles, walked through a per-query-block
// list of kept key blocks.
//
// Persistent kernel, one CTA per SM, work item = (head, 128-row query tile).
// Warp roles (384 threads, three warpgroups):
//   warp 0      TMA producer: the Q tile of each item (double-buffered across
//               items), then K and V of every kept key block into a ring;
//   warp 1      MMA issuer (one thread): S = Q K^T into TMEM (two S buffers,
//               bf16 operands) and O += P V (fp16 operands), P read from
//               TMEM, V from smem;
//   warps 2-3   convert each V tile in shared memory from bf16 to fp16;
//   warps 4-7   softmax of S columns [0, 64), warps 8-11 of [64, 128): one
//               thread per (query row, column half).  The two halves swap
//               their row maxima through shared memory, then each computes
//               fp32 online-softmax weights for its 64 keys with lazy
//               rescaling (O is rescaled only when the running max grows by
//               more than 2^8) and writes them into the S buffer as fp16
//               (11 significant bits; the row sum uses the same rounded
//               values).  In the
//               epilogue each half writes its half of the columns of O / l as
//               bf16 straight from registers to global memory.
// MMA order per item: QK_0, QK_1, PV_0, QK_2, PV_1, ... so the tensor core
// computes S_{j+1} while the softmax works on S_j.
//
// TMEM columns: S buffer b at [128 b, 128 b + 128), O at [256, 256 + d).
// Every mbarrier wait is bounded; a wait that gives up sets
// SVG_DEVICE_TIMEOUT, raises a CTA-wide abort flag and every role drains out.
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "attn.cuh"
#include "common.cuh"
#include "sm100.cuh"

namespace svg {
namespace {

using namespace sm100;

constexpr int kThreads = 384;
constexpr int kBox = 16384;           // one 128-row x 128-byte TMA box
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleLog2 = 8.0f;  // lazy-rescale threshold (factor 256)
constexpr uint32_t kSpinLimit = 1u << 22;
constexpr int kPolyPairs = 7;         // of every 16 exp2 pairs, this many run on the FMA pipe
constexpr int kBarMax = 1;            // named barriers of the 256 softmax threads
constexpr int kBarSum = 2;

template <int D>
struct Cfg {
  static constexpr int kTile = 128 * D * 2;        // bytes of a Q / K / V tile
  static constexpr int kBoxes = D / 64;            // 64-column boxes per tile
  static constexpr int kSlots = D == 64 ? 10 : 4;  // K/V ring entries
  static constexpr int kOffQ = 0;                  // 2 Q buffers
  static constexpr int kOffKV = 2 * kTile;
  // d = 64: the row sums come out of the tensor core as an extra O column:
  // V is extended by a 64-column atom whose first column is 1.0 (fp16)
  static constexpr bool kSumOnTC = D == 64;
  static constexpr int kNO = kSumOnTC ? D + 16 : D;  // O columns (N of P.V)
  static constexpr int kOffOnes = kOffKV + kSlots * kTile;
  static constexpr int kOffRed = kOffOnes + (kSumOnTC ? kBox : 0);  // float [2][2][128] + [2][128]
  static constexpr int kOffBar = kOffRed + 6 * 128 * 4;
  static constexpr int kBars = 2 + 2 + 3 * kSlots + 2 + 2 + 2 + 1;
  static constexpr int kSmem = kOffBar + kBars * 8 + 16 + 1024;  // + alignment slack
  static constexpr uint32_t kIdescQK = idesc_bf16(128, 128, false);
  static constexpr uint32_t kIdescPV = idesc_f16(128, kNO, true);
};

struct Maps {
  CUtensorMap q, k, v;
};

struct Bars {
  uint64_t* q_full;    // [2]
  uint64_t* q_empty;   // [2]
  uint64_t* kv_full;   // [slots]
  uint64_t* kv_empty;  // [slots]
  uint64_t* v_ready;   // [slots] V tile converted to fp16
  uint64_t* s_full;    // [2]
  uint64_t* p_ready;   // [2]
  uint64_t* o_done;    // [2]
  uint64_t* o_free;    // [1]
};

// The list of (bh, qt): [beg, end) into indices, or empty.
__device__ __forceinline__ void item_list(const AttnArgs& a, int bh, int qt, int& beg, int& end,
                                          bool report = false) {
  beg = end = 0;
  const int lid = a.list_id[bh];
  if (lid < 0 || lid >= a.n_lists) {
    if (report) set_status(a.status, SVG_DEVICE_BAD_LIST_ID);
    return;
  }
  const int32_t* ip = a.indptr + static_cast<long long>(lid) * (a.n_qblocks + 1);
  const int b = ip[qt], e = ip[qt + 1];
  if (b < 0 || e < b) {
    if (report) set_status(a.status, SVG_DEVICE_BAD_INDEX);
    return;
  }
  beg = b;
  end = e;
}

__device__ __forceinline__ bool valid_tile(int j, int nb) { return j >= 0 && j < nb; }

// Bounded wait on an mbarrier phase; false if it timed out or another role
// aborted.
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                         int32_t* status) {
  const uint32_t addr = smem_u32(bar);
  for (uint32_t i = 0; i < kSpinLimit; ++i) {
    if (mbar_try_wait(addr, parity)) return true;
    if ((i & 255u) == 255u && *abort_flag) return false;
  }
  *abort_flag = 1;
  set_status(status, SVG_DEVICE_TIMEOUT);
  return false;
}

// 2^t for a pair of arguments on the FMA pipe: t = n + f with n the nearest
// integer (t + 1.5 * 2^23 rounds in the mantissa), 2^f from a degree-4
// minimax polynomial on [-1/2, 1/2] (coefficients fitted for this kernel by
// a Remez iteration; relative error < 3e-6 in fp32), and 2^n added into the
// exponent field.  Arguments are clamped at -40: the fp16 weight of 2^-40 is
// 0 either way.
__device__ __forceinline__ void exp2_poly2(float t0, float t1, float& p0, float& p1) {
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
  constexpr float c0 = 0.9999992847442627f, c1 = 0.6931217908859253f, c2 = 0.240247443318367f,
                  c3 = 0.05591785907745361f, c4 = 0.009570102207362652f;
  t0 = fmaxf(t0, -40.f);
  t1 = fmaxf(t1, -40.f);
  float j0, j1, n0, n1, f0, f1, q0, q1;
  add2(j0, j1, t0, t1, kRound, kRound);
  add2(n0, n1, j0, j1, -kRound, -kRound);
  add2(f0, f1, t0, t1, -n0, -n1);
  fma2(q0, q1, c4, c4, f0, f1, c3, c3);
  fma2(q0, q1, q0, q1, f0, f1, c2, c2);
  fma2(q0, q1, q0, q1, f0, f1, c1, c1);
  fma2(q0, q1, q0, q1, f0, f1, c0, c0);
  p0 = __uint_as_float(__float_as_uint(q0) + (__float_as_uint(j0) << 23));
  p1 = __uint_as_float(__float_as_uint(q1) + (__float_as_uint(j1) << 23));
}

// Softmax of one column half (64 keys) of every S tile, and the matching half
// of the output columns.
template <int D>
__device__ __forceinline__ void softmax_half(const AttnArgs& a, const Bars& B,
                                             volatile int* abort_flag, uint32_t tmem,
                                             float* red_max, float* red_sum, int n_items,
                                             int nb) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int half = (warp >> 2) - 1;  // 0: S columns [0, 64), 1: [64, 128)
  const int quarter = warp & 3;      // TMEM lane quarter this warp may access
  const int row = quarter * 32 + lane;
  const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
  const uint32_t t_o = tmem + lane_off + 256 + half * (D / 2);
  const uint32_t t_sum = tmem + lane_off + 256 + D;  // row-sum column (d = 64)
  const float sl2 = a.scale * kLog2e;
  const int N = a.N;
  uint32_t g = 0;  // tiles so far
  bool ok = true;
  for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
    const int bh = item / nb, qt = item - bh * nb;
    int beg, end;
    item_list(a, bh, qt, beg, end);
    float m_used = -INFINITY, l = 0.f;
    bool first = true;
    for (int e = beg; e < end && ok; ++e) {
      const int j = a.indices[e];
      if (!valid_tile(j, nb)) continue;
      const int sb = g & 1;
      if (!(ok = wait_bar(&B.s_full[sb], (g >> 1) & 1, abort_flag, a.status))) break;
      tc_fence_after();
      const uint32_t t_s = tmem + lane_off + sb * 128;
      float s[64];
      {
        uint32_t r0[32], r1[32];
        tmem_ld32(t_s + 64 * half, r0);
        tmem_ld32(t_s + 64 * half + 32, r1);
        tmem_wait_ld();
        reg_fence32(r0);
        reg_fence32(r1);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          s[i] = __uint_as_float(r0[i]);
          s[32 + i] = __uint_as_float(r1[i]);
        }
      }
      const int valid_cols = min(128, N - j * 128) - 64 * half;
      if (valid_cols < 64) {
#pragma unroll
        for (int i = 0; i < 64; ++i)
          if (i >= valid_cols) s[i] = -INFINITY;
      }
      float mx4[4] = {s[0], s[1], s[2], s[3]};
#pragma unroll
      for (int i = 4; i < 60; i += 8) {  // s[4 .. 59]
#pragma unroll
        for (int c = 0; c < 4; ++c) mx4[c] = max3(mx4[c], s[i + c], s[i + 4 + c]);
      }
      float mx = max3(max3(mx4[0], mx4[1], s[60]), max3(mx4[2], mx4[3], s[61]),
                      fmaxf(s[62], s[63]));
      // both halves have read all of S once they pass this barrier, so the P
      // writes below cannot overwrite scores the other half still needs
      float* rm = red_max + (sb * 2) * 128;
      rm[half * 128 + row] = mx;
      named_bar_sync(kBarMax, 256);
      mx = fmaxf(mx, rm[(half ^ 1) * 128 + row]);
      const float tm = mx * sl2;
      if (first) {
        m_used = tm;
      } else {
        const bool need = tm > m_used + kRescaleLog2;
        if (__any_sync(0xffffffffu, need)) {
          // O must hold PV of the previous tile before it is rescaled
          if (!(ok = wait_bar(&B.o_done[(g - 1) & 1], ((g - 1) >> 1) & 1, abort_flag, a.status)))
            break;
          tc_fence_after();
          const float m_new = need ? tm : m_used;
          const float alpha = exp2f(m_used - m_new);
          uint32_t r[32];
#pragma unroll
          for (int ch = 0; ch < D / 64; ++ch) {
            tmem_ld32(t_o + ch * 32, r);
            tmem_wait_ld();
            reg_fence32(r);
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
            tmem_st32(t_o + ch * 32, r);
            tmem_wait_st();  // r is reused by the next chunk
          }
          if constexpr (Cfg<D>::kSumOnTC) {
            if (half == 1) {  // the row-sum columns [D, D + 16)
              uint32_t r16[16];
              tmem_ld16(t_sum, r16);
              tmem_wait_ld();
              reg_fence16(r16);
#pragma unroll
              for (int i = 0; i < 16; ++i) r16[i] = __float_as_uint(__uint_as_float(r16[i]) * alpha);
              tmem_st16(t_sum, r16);
              tmem_wait_st();
            }
          } else {
            l *= alpha;
          }
          m_used = m_new;
        }
      }
      const float neg = -m_used;
      float lx = 0.f, ly = 0.f;
#pragma unroll
      for (int q2 = 0; q2 < 2; ++q2) {
        uint32_t ph[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float t0, t1, p0, p1;
          fma2(t0, t1, s[32 * q2 + 2 * i], s[32 * q2 + 2 * i + 1], sl2, sl2, neg, neg);
          if ((i & 1) == 0 && i < 2 * kPolyPairs) {
            exp2_poly2(t0, t1, p0, p1);  // FMA pipe
          } else {
            p0 = fast_exp2(t0);  // MUFU
            p1 = fast_exp2(t1);
          }
          const __half2 h = __floats2half2_rn(p0, p1);
          ph[i] = *reinterpret_cast<const uint32_t*>(&h);
          if constexpr (!Cfg<D>::kSumOnTC) {
            // the row sum uses the fp16-rounded weights the MMA sees
            const float2 r = __half22float2(h);
            add2(lx, ly, lx, ly, r.x, r.y);
          }
        }
        // P column c (fp16 pair) holds keys 2c, 2c+1
        tmem_st16(t_s + 32 * half + 16 * q2, ph);
        tmem_wait_st();  // ph is rewritten by the next quarter
      }
      if constexpr (!Cfg<D>::kSumOnTC) l += lx + ly;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&B.p_ready[sb]);
      first = false;
      ++g;
    }
    if (!ok) break;
    // -------------------------------------------------------------- epilogue
    const bool empty = first;
    float ltot = 0.f;
    if (!empty) {
      if (!(ok = wait_bar(&B.o_done[(g - 1) & 1], ((g - 1) >> 1) & 1, abort_flag, a.status)))
        break;
      tc_fence_after();
      if constexpr (Cfg<D>::kSumOnTC) {
        uint32_t r1 = tmem_ld1(t_sum);
        tmem_wait_ld();
        reg_fence1(r1);
        ltot = __uint_as_float(r1);
      } else {
        red_sum[half * 128 + row] = l;
        named_bar_sync(kBarSum, 256);
        ltot = l + red_sum[(half ^ 1) * 128 + row];
      }
    }
    const float inv = ltot > 0.f ? 1.f / ltot : 0.f;
    const int n = qt * 128 + row;
    __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(a.o) +
                          (static_cast<long long>(bh) * N + n) * D + half * (D / 2);
#pragma unroll
    for (int ch = 0; ch < D / 64; ++ch) {
      uint32_t r[32];
      if (!empty) {
        tmem_ld32(t_o + ch * 32, r);
        tmem_wait_ld();
        reg_fence32(r);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) r[i] = 0u;
      }
      if (n < N) {
#pragma unroll
        for (int c16 = 0; c16 < 4; ++c16) {
          uint4 v;
          v.x = pack_bf16x2(__uint_as_float(r[8 * c16 + 0]) * inv,
                            __uint_as_float(r[8 * c16 + 1]) * inv);
          v.y = pack_bf16x2(__uint_as_float(r[8 * c16 + 2]) * inv,
                            __uint_as_float(r[8 * c16 + 3]) * inv);
          v.z = pack_bf16x2(__uint_as_float(r[8 * c16 + 4]) * inv,
                            __uint_as_float(r[8 * c16 + 5]) * inv);
          v.w = pack_bf16x2(__uint_as_float(r[8 * c16 + 6]) * inv,
                            __uint_as_float(r[8 * c16 + 7]) * inv);
          *reinterpret_cast<uint4*>(orow + ch * 32 + c16 * 8) = v;
        }
      }
    }
    if (!empty) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(B.o_free);
    }
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_sm100_kernel(const __grid_constant__ Maps maps, const AttnArgs a) {
  using C = Cfg<D>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bar_base = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  Bars B;
  B.q_full = bar_base;
  B.q_empty = bar_base + 2;
  B.kv_full = bar_base + 4;
  B.kv_empty = B.kv_full + C::kSlots;
  B.v_ready = B.kv_empty + C::kSlots;
  B.s_full = B.v_ready + C::kSlots;
  B.p_ready = B.s_full + 2;
  B.o_done = B.p_ready + 2;
  B.o_free = B.o_done + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(B.o_free + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* red_max = reinterpret_cast<float*>(smem + C::kOffRed);  // [S buffer][half][row]
  float* red_sum = red_max + 4 * 128;                             // [half][row]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int N = a.N, nb = n_tiles(N);
  const int n_items = a.B * a.H * nb;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&B.q_full[i], 1);
      mbar_init(&B.q_empty[i], 1);
      mbar_init(&B.s_full[i], 1);
      mbar_init(&B.p_ready[i], 8);
      mbar_init(&B.o_done[i], 1);
    }
    for (int i = 0; i < C::kSlots; ++i) {
      mbar_init(&B.kv_full[i], 1);
      mbar_init(&B.kv_empty[i], 1);
      mbar_init(&B.v_ready[i], 2);
    }
    mbar_init(B.o_free, 8);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&maps.q);
    prefetch_tmap(&maps.k);
    prefetch_tmap(&maps.v);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  if (C::kSumOnTC && (warp == 2 || warp == 3)) {
    // 128 rows x 64 fp16 columns, swizzled like a V box: column 0 = 1.0
    uint4* ones = reinterpret_cast<uint4*>(smem + C::kOffOnes);
    for (int r = threadIdx.x - 64; r < 128; r += 64)
#pragma unroll
      for (int cc = 0; cc < 8; ++cc)
        ones[r * 8 + cc] = make_uint4(cc == (r & 7) ? 0x3C00u : 0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tmem_s0 = tmem, tmem_o = tmem + 256;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t L = 0, c = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
        const int bh = item / nb, qt = item - bh * nb;
        int beg, end;
        item_list(a, bh, qt, beg, end, true);
        int first = beg;
        while (first < end && !valid_tile(a.indices[first], nb)) {
          set_status(a.status, SVG_DEVICE_BAD_INDEX);
          ++first;
        }
        if (first == end) continue;
        const int qb = c & 1;
        if (!(ok = wait_bar(&B.q_empty[qb], ((c >> 1) & 1) ^ 1, abort_flag, a.status))) break;
        mbar_arrive_expect_tx(&B.q_full[qb], C::kTile);
        for (int bx = 0; bx < C::kBoxes; ++bx)
          tma_load_3d(smem + C::kOffQ + qb * C::kTile + bx * kBox, &maps.q, &B.q_full[qb], 64 * bx,
                      qt * 128, bh);
        for (int e = first; e < end && ok; ++e) {
          const int j = a.indices[e];
          if (!valid_tile(j, nb)) {
            set_status(a.status, SVG_DEVICE_BAD_INDEX);
            continue;
          }
          for (int t = 0; t < 2; ++t, ++L) {
            const int slot = L % C::kSlots;
            if (!(ok = wait_bar(&B.kv_empty[slot], ((L / C::kSlots) & 1) ^ 1, abort_flag,
                                a.status)))
              break;
            mbar_arrive_expect_tx(&B.kv_full[slot], C::kTile);
            const CUtensorMap* m = t == 0 ? &maps.k : &maps.v;
            for (int bx = 0; bx < C::kBoxes; ++bx)
              tma_load_3d(smem + C::kOffKV + slot * C::kTile + bx * kBox, m, &B.kv_full[slot],
                          64 * bx, j * 128, bh);
          }
        }
        ++c;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t L = 0, g = 0, c = 0;
      bool ok = true;
      auto issue_pv = [&](uint32_t gp, uint32_t lv, bool first_of_item) -> bool {
        const int sb = gp & 1;
        if (!wait_bar(&B.p_ready[sb], (gp >> 1) & 1, abort_flag, a.status)) return false;
        if (first_of_item && c > 0 && !wait_bar(B.o_free, (c - 1) & 1, abort_flag, a.status))
          return false;
        const int slot = lv % C::kSlots;
        if (!wait_bar(&B.v_ready[slot], (lv / C::kSlots) & 1, abort_flag, a.status)) return false;
        tc_fence_after();
        const uint32_t vbase = smem_u32(smem + C::kOffKV + slot * C::kTile);
        // second 64-column atom of B: V columns 64.. (d = 128) or the ones
        // column that accumulates the row sums (d = 64)
        const uint32_t lbo = C::kSumOnTC ? smem_u32(smem + C::kOffOnes) - vbase : kBox;
        // O (+)= P V, P (fp16) in S columns [0, 64), V converted to fp16
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tmem_o, tmem_s0 + sb * 128 + kk * 8, sdesc_sw128(vbase + kk * 2048, lbo, 1024),
                 C::kIdescPV, (first_of_item && kk == 0) ? 0u : 1u);
        tc_commit(&B.kv_empty[slot]);
        tc_commit(&B.o_done[sb]);
        return true;
      };
      for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
        const int bh = item / nb, qt = item - bh * nb;
        int beg, end;
        item_list(a, bh, qt, beg, end);
        bool any = false;
        for (int e = beg; e < end && !any; ++e) any = valid_tile(a.indices[e], nb);
        if (!any) continue;
        const int qb = c & 1;
        if (!(ok = wait_bar(&B.q_full[qb], (c >> 1) & 1, abort_flag, a.status))) break;
        const uint32_t qbase = smem_u32(smem + C::kOffQ + qb * C::kTile);
        bool have_pending = false, pending_first = false;
        uint32_t pend_g = 0, pend_lv = 0;
        bool first = true;
        for (int e = beg; e < end && ok; ++e) {
          if (!valid_tile(a.indices[e], nb)) continue;
          const int slot = L % C::kSlots;
          if (!(ok = wait_bar(&B.kv_full[slot], (L / C::kSlots) & 1, abort_flag, a.status))) break;
          tc_fence_after();
          const int sb = g & 1;
          const uint32_t kbase = smem_u32(smem + C::kOffKV + slot * C::kTile);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * kBox + (kk & 3) * 32;
            mma_ss(tmem_s0 + sb * 128, sdesc_sw128(qbase + off, 16, 1024),
                   sdesc_sw128(kbase + off, 16, 1024), C::kIdescQK, kk > 0 ? 1u : 0u);
          }
          tc_commit(&B.s_full[sb]);
          tc_commit(&B.kv_empty[slot]);
          if (have_pending && !(ok = issue_pv(pend_g, pend_lv, pending_first))) break;
          have_pending = true;
          pending_first = first;
          pend_g = g;
          pend_lv = L + 1;
          L += 2;
          ++g;
          first = false;
        }
        if (!ok) break;
        tc_commit(&B.q_empty[qb]);  // Q buffer free once its last QK^T completes
        if (!(ok = issue_pv(pend_g, pend_lv, pending_first))) break;
        ++c;
      }
    }
  } else if (warp == 2 || warp == 3) {
    // ------------------------------------------------------------ V to fp16
    // Converts every V tile in place, in the order the MMA issuer consumes
    // them.  bf16 -> fp16 is exact for |v| <= 65504 (fp16 subnormals keep
    // the absolute error below 2^-25); larger values become inf and are
    // reported as SVG_DEVICE_RANGE.
    const int t = threadIdx.x - 64;  // 0..63
    uint32_t L = 0;
    bool ok = true, range = false;
    for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
      const int bh = item / nb, qt = item - bh * nb;
      int beg, end;
      item_list(a, bh, qt, beg, end);
      for (int e = beg; e < end && ok; ++e) {
        if (!valid_tile(a.indices[e], nb)) continue;
        const uint32_t lv = L + 1;
        const int slot = lv % C::kSlots;
        if (!(ok = wait_bar(&B.kv_full[slot], (lv / C::kSlots) & 1, abort_flag, a.status))) break;
        uint4* tile = reinterpret_cast<uint4*>(smem + C::kOffKV + slot * C::kTile);
#pragma unroll 4
        for (int c = t; c < C::kTile / 16; c += 64) {
          uint4 v = tile[c];
          uint32_t* w = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float lo = __uint_as_float(w[i] << 16), hi = __uint_as_float(w[i] & 0xffff0000u);
            range |= fabsf(lo) > 65504.f || fabsf(hi) > 65504.f;
            const __half2 h = __floats2half2_rn(lo, hi);
            w[i] = *reinterpret_cast<const uint32_t*>(&h);
          }
          tile[c] = v;
        }
        fence_proxy_async_smem();  // generic-proxy writes -> tensor-core reads
        __syncwarp();
        if (lane == 0) mbar_arrive(&B.v_ready[slot]);
        L += 2;
      }
    }
    if (__any_sync(0xffffffffu, range) && lane == 0) set_status(a.status, SVG_DEVICE_RANGE);
  } else if (warp >= 4) {
    softmax_half<D>(a, B, abort_flag, tmem, red_max, red_sum, n_items, nb);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------ host side

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// [B*H][N][d] bf16 viewed as a 3-D tensor (d, N, B*H); box 64 x 128 x 1,
// 128-byte swizzle.  Rows beyond N are zero-filled on load.
bool make_map(CUtensorMap* m, const void* base, int BH, int N, int d) {
  auto enc = get_encode();
  if (enc == nullptr) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                        static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(N) * d * 2};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

}  // namespace

template <int D>
svg_status launch_attn_sm100(const AttnArgs& a, cudaStream_t s) {
  using C = Cfg<D>;
  Maps maps;
  const int BH = a.B * a.H;
  if (!make_map(&maps.q, a.q, BH, a.N, D) || !make_map(&maps.k, a.k, BH, a.N, D) ||
      !make_map(&maps.v, a.v, BH, a.N, D))
    return fail(SVG_ERR_CUDA, "sparse_attn: cannot encode TMA descriptors");
  if (cudaFuncSetAttribute(attn_sm100_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           C::kSmem) != cudaSuccess)
    return fail(SVG_ERR_CUDA, "sparse_attn: cannot reserve %d bytes of shared memory", C::kSmem);
  const long long items = static_cast<long long>(BH) * n_tiles(a.N);
  const int grid = static_cast<int>(items < sm_count() ? items : sm_count());
  attn_sm100_kernel<D><<<grid, kThreads, C::kSmem, s>>>(maps, a);
  return check_launch("sparse_attn sm100");
}

template svg_status launch_attn_sm100<64>(const AttnArgs&, cudaStream_t);
template svg_status launch_attn_sm100<128>(const AttnArgs&, cudaStream_t);

}  // namespace svg
