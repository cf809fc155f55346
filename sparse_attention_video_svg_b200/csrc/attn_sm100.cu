// Block-sparse attention on the B200 tensor core (tcgen05 + TMEM + TMA).
//
// Video-diffusion acceleration survey (wmrh.cn/news/48564), section 2.1:
// o = softmax(Q K^T / sqrt(d_k)) V; section 5.3: tiled on chip with an online
// softmax.  CalibAtt article (lpnh.cn/news/568491), sections 2.2 and 3.3:
// keep/skip decisions on 128 x 128 tiles, walked through a per-query-block
// list of kept key blocks.
//
// Persistent kernel, one CTA per SM.  A work item is a pair of adjacent
// 128-row query tiles of one head (members 0 and 1).  The producer walks the
// two members' key lists as one merged sequence of steps, so a key block that
// both keep is loaded once and feeds both; each member then runs its own
// pipeline on the tensor core.
// Warp roles (384 threads, three warpgroups):
//   warp 0      TMA producer: each member's Q tile, then K and V of every
//               step into a ring, with a step record (which members keep the
//               block, item boundaries, the head's V exponent) in shared
//               memory;
//   d = 64:  warps 1, 2 MMA issuers of members 0 and 1 (one thread each),
//               warp 3 the V converter;
//   d = 128: warp 1 the one MMA issuer of both members (order on the tensor
//               core: P.V of member 0, Q K^T of member 0, P.V of member 1,
//               Q K^T of member 1), warps 2 and 3 the V converters (half a
//               tile each);
//               S_t = Q_t K^T into TMEM (bf16 operands) and O_t += P_t V
//               (fp16 operands, P_t read from TMEM, V from smem).  A K/V ring
//               entry is released when every issuer has passed it;
//   converters  each V tile in shared memory from bf16 to fp16, scaled by
//               2^-e with the head's V exponent e (0 unless |v| > 65504 occurs
//               in the head), so any finite bf16 V is exact in fp16;
//   warps 4-7   softmax of member 0, warps 8-11 of member 1: one thread per
//               query row holds the tile's 128 scores, fp32 online softmax
//               with lazy rescaling (O is rescaled only when the running max
//               grows by more than 2^8); the weights go to TMEM as fp16
//               (11 significant bits) and the row sums add the same rounded
//               values (mixed-precision adds).  The epilogue writes
//               O * 2^e / l as bf16 from registers.
// Every exponential runs on the MUFU (ex2.approx): FMA-pipe work in the
// softmax warps measurably slows the issue of the tensor-core instructions,
// so the softmax keeps its FMA-pipe share small.  Each tile's MMAs are
// issued from one asm block (about two instructions per MMA).
// d = 64: P_t has TMEM columns of its own, so the next S_t = Q_t K^T is
// issued as soon as the softmax has read S_t and runs during the softmax.
// d = 128 (TMEM is full with two S and two O): P_t overwrites S_t, and the
// next Q_t K^T is issued after O_t += P_t V; tcgen05 operations of one thread
// complete in issue order, so "S_t full" also means that P.V finished.
//
// Every mbarrier wait is bounded; a wait that gives up sets
// SVG_DEVICE_TIMEOUT, raises a CTA-wide abort flag and every role drains out.
#include <cuda_fp16.h>
#include <cudaTypedefs.h>
#include <limits.h>

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
constexpr uint32_t kDrainLimit = 1u << 20;
constexpr int kLaunchRegs = 168;      // 65536 / 384, rounded down to a multiple of 8

template <int D>
struct Cfg {
  static constexpr int kTile = 128 * D * 2;        // bytes of a Q / K / V tile
  static constexpr int kBoxes = D / 64;            // 64-column boxes per tile
  static constexpr int kQDepth = D == 64 ? 2 : 1;  // Q buffers per member
  // K/V ring entries; even, so K tiles always sit in even and V tiles in odd
  // entries
  static constexpr int kSlots = D == 64 ? 8 : 4;
  static constexpr int kSteps = kSlots / 2;        // merged-walk steps in the ring
  // Step records in flight.  K and V entries are claimed one at a time, so
  // the producer may run up to kSteps + 1 steps ahead of the slowest reader
  // of a record (the converter): kSteps + 2 records are live at most.
  static constexpr int kInfo = 8;
  static_assert(kInfo >= kSteps + 2, "step records");
  static constexpr bool kSepP = D == 64;           // P_t in TMEM columns of its own
  // d = 128: one MMA issuer for both members (warp 1), which fixes the
  // order on the tensor core, and two V converter warps (2, 3); d = 64: one
  // issuer per member (warps 1, 2) and one converter (warp 3)
  static constexpr bool kOneIssuer = D == 128;
  static constexpr int kConvWarps = kOneIssuer ? 2 : 1;
  static constexpr int kOffQ = 0;                  // [member][depth]
  static constexpr int kOffKV = 2 * kQDepth * kTile;
  static constexpr int kOffInfo = kOffKV + kSlots * kTile;  // uint32 [kInfo]
  static constexpr int kOffBar = kOffInfo + 64;
  static constexpr int kBars = 4 * kQDepth + 3 * kSlots + 5 * 2;
  static constexpr int kSmem = kOffBar + kBars * 8 + 16 + 1024;  // + alignment slack
  // TMEM columns
  static constexpr uint32_t kColS = 0;                   // S_t at 128 t
  static constexpr uint32_t kColP = kSepP ? 256 : 0;     // P_t at kColP + kPStride t
  static constexpr uint32_t kPStride = kSepP ? 64 : 128;
  static constexpr uint32_t kColO = kSepP ? 384 : 256;   // O_t at kColO + kOStride t
  static constexpr uint32_t kOStride = kSepP ? 64 : 128;
  // Register split of the 384 x 168 launch registers: warpgroup 0
  // (producer, MMA issuers, converter) drops to kRegsLow, the two softmax
  // warpgroups rise to kRegsHigh (the split with the fewest spills ptxas reports).
  static constexpr int kRegsLow = D == 128 ? 72 : 88;
  static constexpr int kRegsHigh = D == 128 ? 216 : 208;
  static_assert(128 * kRegsLow + 256 * kRegsHigh <= kThreads * kLaunchRegs, "register split");
  static constexpr uint32_t kIdescQK = idesc_bf16(128, 128, false);
  static constexpr uint32_t kIdescPV = idesc_f16(128, D, true);
  static_assert(kSlots % 2 == 0, "K and V must alternate between even and odd ring entries");
  static_assert(kSmem <= 227 * 1024, "shared memory budget");
  static_assert(kColO + 2 * kOStride <= 512, "TMEM budget");
};

struct Maps {
  CUtensorMap q, k, v;
  CUtensorMap qt, kt, vt;  // token-major copies (encoded only when given)
};

struct Bars {
  uint64_t* q_full;    // [2][depth]
  uint64_t* q_empty;   // [2][depth]
  uint64_t* kv_full;   // [slots]
  uint64_t* kv_empty;  // [slots] one commit from each member's issuer
  uint64_t* v_ready;   // [slots] V tile converted to fp16
  uint64_t* s_full;    // [2] S_t written
  uint64_t* s_free;    // [2] S_t read by the softmax (4 warps; separate-P layout)
  uint64_t* p_ready;   // [2] P_t written (4 warps)
  uint64_t* o_done;    // [2] O_t += P_t V finished
  uint64_t* drain;     // [2] every MMA of an issuer finished
};

__device__ __forceinline__ bool valid_tile(int j, int nb) { return j >= 0 && j < nb; }

// Step record the producer publishes with each K/V pair: bits 0-1 the members
// that keep the block, bits 2-3 the members for which it is the first block
// of the item, bits 4-5 the last; bit 6 marks the end (no tile loaded).
constexpr uint32_t kStepEnd = 1u << 6;
constexpr uint32_t kStepGathered = 1u << 7;  // Q / K / V of this step came through cp.async
// bits 8-15: the head's V exponent e (v * 2^-e is converted; 0 = unscaled)
constexpr int kStepExpShift = 8;

// The V exponent the kernel applies to head bh: svg_v_exponents' value when
// it is a usable scale (1 .. 126), else 0 (no exponents given, a head that
// already fits fp16, or 255 for inf / NaN, which no scale fixes).
__device__ __forceinline__ uint32_t v_exponent(const AttnArgs& a, int bh) {
  if (a.v_exp == nullptr) return 0;
  const int e = a.v_exp[bh];
  return (e > 0 && e < 127) ? static_cast<uint32_t>(e) : 0u;
}

// Entries [beg, end) of `indices` for query tile qt of head bh; empty for a
// tile past the end or a bad list.
__device__ __forceinline__ void member_list(const AttnArgs& a, int bh, int qt, int nb, int& beg,
                                            int& end, bool report) {
  beg = end = 0;
  if (qt < 0 || qt >= nb) return;
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

// A list entry is used when it is a valid key block above the member's last
// used one: rows must be strictly ascending, and an out-of-range, repeated or
// descending entry is skipped (and reported), so a key block is never
// attended twice.  The softmax warps apply the same rule to the same list.
__device__ __forceinline__ bool usable(int j, int last, int nb) { return valid_tile(j, nb) && j > last; }

__device__ __forceinline__ void skip_invalid(const AttnArgs& a, int nb, int& p, int e, int last,
                                             bool report) {
  while (p < e && !usable(a.indices[p], last, nb)) {
    if (report) set_status(a.status, SVG_DEVICE_BAD_INDEX);
    ++p;
  }
}

// Next key block of the merged walk over both members' lists, whose heads
// are usable (or exhausted).  mask bit t: member t keeps block j.  Every
// usable entry of either list is visited exactly once, in ascending order;
// equal heads are shared.  Afterwards both heads are again usable or
// exhausted.
__device__ __forceinline__ bool merge_next(const AttnArgs& a, int nb, int (&p)[2],
                                           const int (&e)[2], int& j, int& mask, bool report) {
  int jj[2];
#pragma unroll
  for (int t = 0; t < 2; ++t) jj[t] = p[t] < e[t] ? a.indices[p[t]] : INT_MAX;
  j = min(jj[0], jj[1]);
  if (j == INT_MAX) return false;
  mask = (jj[0] == j ? 1 : 0) | (jj[1] == j ? 2 : 0);
#pragma unroll
  for (int t = 0; t < 2; ++t)
    if (mask >> t & 1) {
      ++p[t];
      skip_invalid(a, nb, p[t], e[t], j, report);
    }
  return true;
}

// Bounded wait on an mbarrier phase; false if it timed out or another role
// aborted (checked every 256 polls).  SW (a launch whose svg_set_wait_limit
// differs from the default) reads the poll limit from the shared word after
// the CTA's abort flag; otherwise the limit is the compile-time default.
template <bool SW>
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                         int32_t* status) {
  const uint32_t addr = smem_u32(bar);
  const uint32_t limit = SW ? static_cast<uint32_t>(abort_flag[1]) : kDefaultWaitLimit;
  for (uint32_t i = 0; i < limit; ++i) {
    if (mbar_try_wait(addr, parity)) return true;
    if ((i & 255u) == 255u && *abort_flag) return false;
  }
  *abort_flag = 1;
  set_status(status, SVG_DEVICE_TIMEOUT);
  return false;
}

// Bounded wait that ignores the abort flag (used to drain copies and MMAs in
// flight before the CTA exits).
__device__ __forceinline__ void drain_bar(uint64_t* bar, uint32_t parity) {
  const uint32_t addr = smem_u32(bar);
  for (uint32_t i = 0; i < kDrainLimit; ++i)
    if (mbar_try_wait(addr, parity)) return;
}

// Softmax and epilogue of member t (warps 4 + 4t .. 7 + 4t).
template <int D, bool SW>
__device__ __forceinline__ void softmax_member(const AttnArgs& a, const Bars& B,
                                               volatile int* abort_flag, uint32_t tmem,
                                               int n_items, int n_pairs, int nb) {
  using C = Cfg<D>;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = (warp - 4) >> 2;  // member
  const int quarter = warp & 3;   // TMEM lane quarter this warp may access
  const int row = quarter * 32 + lane;
  const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
  const uint32_t t_s = tmem + lane_off + C::kColS + 128 * t;
  const uint32_t t_p = tmem + lane_off + C::kColP + C::kPStride * t;
  const uint32_t t_o = tmem + lane_off + C::kColO + C::kOStride * t;
  const float sl2 = a.scale * kLog2e;
  const int N = a.N;
  uint32_t g = 0;  // tiles of this member so far
  bool ok = true;
  for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
    const int bh = item / n_pairs;
    const int qt = query_tile(a, bh, 2 * (item - bh * n_pairs) + t, nb);
    if (qt < 0) continue;
    int beg, end;
    member_list(a, bh, qt, nb, beg, end, false);
    float m_used = -INFINITY, l = 0.f;
    bool first = true;
    int last = -1;
    for (int e = beg; e < end; ++e) {
      const int j = a.indices[e];
      if (!usable(j, last, nb)) continue;
      last = j;
      if (!(ok = wait_bar<SW>(&B.s_full[t], g & 1, abort_flag, a.status))) break;
      tc_fence_after();
      float s[128];
      {
        uint32_t r[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(t_s + 32 * c, r[c]);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          reg_fence32(r[c]);
#pragma unroll
          for (int i = 0; i < 32; ++i) s[32 * c + i] = __uint_as_float(r[c][i]);
        }
      }
      if constexpr (C::kSepP) {
        // S_t is in registers: the next Q_t K^T may overwrite it
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&B.s_free[t]);
      }
      const int valid_cols = min(128, N - j * 128);
      if (valid_cols < 128) {
#pragma unroll
        for (int i = 0; i < 128; ++i)
          if (i >= valid_cols) s[i] = -INFINITY;
      }
      float mx4[4] = {s[0], s[1], s[2], s[3]};
#pragma unroll
      for (int i = 4; i < 124; i += 8) {  // s[4 .. 123]
#pragma unroll
        for (int c = 0; c < 4; ++c) mx4[c] = max3(mx4[c], s[i + c], s[i + 4 + c]);
      }
      const float mx = max3(max3(mx4[0], s[124], s[125]), max3(mx4[1], s[126], s[127]),
                            fmaxf(mx4[2], mx4[3]));
      const float tm = mx * sl2;
      float alpha = 1.f;
      bool rescale = false;
      if (first) {
        m_used = tm;
      } else {
        const bool need = tm > m_used + kRescaleLog2;
        if (__any_sync(0xffffffffu, need)) {
          rescale = true;
          const float m_new = need ? tm : m_used;
          alpha = exp2f(m_used - m_new);
          m_used = m_new;
        }
      }
      const float neg = -m_used;
      float lx = 0.f, ly = 0.f;
      uint32_t ph[4][16];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float t0, t1, p0, p1;
          fma2(t0, t1, s[32 * c + 2 * i], s[32 * c + 2 * i + 1], sl2, sl2, neg, neg);
          p0 = fast_exp2(t0);
          p1 = fast_exp2(t1);
          const __half2 h = __floats2half2_rn(p0, p1);
          ph[c][i] = *reinterpret_cast<const uint32_t*>(&h);
          // the row sum uses the fp16-rounded weights the MMA sees (an fp32
          // sum of the unrounded weights is faster, but leaves the output off
          // by up to ~2e-4 of |o|, beyond the bf16 tolerance at |o| >= 8)
          add_f16x2_to_f32(lx, ly, ph[c][i]);
        }
      }
      if constexpr (C::kSepP) {
        // P_t and O_t are free once the previous P.V of this member is done
        // (waited for only now, so that P.V overlaps the exponentials)
        if (g > 0) {
          if (!(ok = wait_bar<SW>(&B.o_done[t], (g - 1) & 1, abort_flag, a.status))) break;
          tc_fence_after();
        }
      }
      // (separate-P layout off: S_t full implies every earlier P.V of this
      // member has completed)
      // P column 16 c + i (fp16 pair) holds keys 32 c + 2 i, 32 c + 2 i + 1
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_st16(t_p + 16 * c, ph[c]);
      if (rescale) {
        uint32_t r[32];
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
          tmem_ld32(t_o + ch * 32, r);
          tmem_wait_ld();
          reg_fence32(r);
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
          tmem_st32(t_o + ch * 32, r);
        }
      }
      l = l * alpha + (lx + ly);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&B.p_ready[t]);
      first = false;
      ++g;
    }
    if (!ok) break;
    // -------------------------------------------------------------- epilogue
    const bool empty = first;
    float inv = 0.f;
    if (!empty) {
      if (!(ok = wait_bar<SW>(&B.o_done[t], (g - 1) & 1, abort_flag, a.status))) break;
      tc_fence_after();
      // 1 / l, times 2^e for a head whose V was converted as v * 2^-e
      inv = l > 0.f ? 1.f / l : 0.f;
      const uint32_t e = v_exponent(a, bh);
      if (e) inv *= __uint_as_float((127u + e) << 23);
    }
    const int n = qt * 128 + row;
    // token-major heads over frame-major memory write row n back to its frame-major place
    const int nm = (scatters_output(a, bh) && n < N) ? token_major_row(n, a.frames, a.tokens_per_frame) : n;
    __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(a.o) + (static_cast<long long>(bh) * N + nm) * D;
#pragma unroll
    for (int ch = 0; ch < D / 32; ch += 2) {
      uint32_t r[2][32];
      if (!empty) {
        tmem_ld32(t_o + ch * 32, r[0]);
        tmem_ld32(t_o + ch * 32 + 32, r[1]);
        tmem_wait_ld();
        reg_fence32(r[0]);
        reg_fence32(r[1]);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) r[0][i] = r[1][i] = 0u;
      }
      if (n < N) {
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int c16 = 0; c16 < 4; ++c16) {
            const uint32_t* x = &r[h][8 * c16];
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(x[0]) * inv, __uint_as_float(x[1]) * inv);
            v.y = pack_bf16x2(__uint_as_float(x[2]) * inv, __uint_as_float(x[3]) * inv);
            v.z = pack_bf16x2(__uint_as_float(x[4]) * inv, __uint_as_float(x[5]) * inv);
            v.w = pack_bf16x2(__uint_as_float(x[6]) * inv, __uint_as_float(x[7]) * inv);
            *reinterpret_cast<uint4*>(orow + (ch + h) * 32 + c16 * 8) = v;
          }
      }
    }
    // the next item's first P.V (accumulate off) is issued after this
    // member's next p_ready, which follows these TMEM reads in program order
  }
}

// 128 token-major rows m0 .. m0 + 127 of one head's frame-major [N][D]
// matrix (row m is memory row (m mod F) P + m div F), copied by the 32 lanes
// of a warp into a tile laid out exactly like the 128-byte-swizzled TMA
// boxes (box bx holds columns 64 bx .. 64 bx + 63; the 16-byte chunk c of
// row r sits at chunk position c ^ (r mod 8)).  Rows at or past N are
// zero-filled.
template <int D>
__device__ __forceinline__ void gather_rows(unsigned char* dst, const __nv_bfloat16* src, int m0,
                                            int N, int F, int P) {
  constexpr int CH = D / 8;       // 16-byte chunks per row
  constexpr int RSTEP = 32 / CH;  // rows between one lane's copies
  const int lane = threadIdx.x & 31;
  const int c = lane % CH;
  int r = lane / CH;
  int m = m0 + r;
  int f = m % F, sp = m / F;  // m = sp * F + f
#pragma unroll 4
  for (; r < 128; r += RSTEP) {
    const bool ok = m < N;
    const long long n = ok ? static_cast<long long>(f) * P + sp : 0;
    cp_async16(dst + (c >> 3) * kBox + r * 128 + (((c & 7) ^ (r & 7)) << 4), src + n * D + c * 8,
               ok);
    m += RSTEP;
    f += RSTEP;
    while (f >= F) {
      f -= F;
      ++sp;
    }
  }
}

// TMA producer (warp 0, all lanes): Q tiles and the merged walk's K / V
// tiles.  Heads in memory order load with TMA; heads that run token-major
// over frame-major memory gather their rows with cp.async: every lane hands
// its copies to the tile's mbarrier (cp.async.mbarrier.arrive) and the leader
// adds the phase's regular arrival, so the barrier completes when the rows
// have landed.  The consumers fence the async proxy after their wait, as the
// tensor core reads what the generic proxy wrote.
template <int D, bool SW>
__device__ __forceinline__ void producer(const AttnArgs& a, const Maps& maps, const Bars& B,
                                         unsigned char* smem, volatile uint32_t* step_info,
                                         volatile int* abort_flag, int n_items, int n_pairs,
                                         int nb) {
  using C = Cfg<D>;
  constexpr int QD = C::kQDepth, S = C::kSlots;
  const int lane = threadIdx.x & 31;
  const bool leader = lane == 0;
  const int N = a.N, F = a.frames, P = a.tokens_per_frame;
  uint32_t L = 0, cq[2] = {0, 0};
  bool ok = true;
  auto leader_wait = [&](uint64_t* bar, uint32_t parity) -> bool {
    int r = 1;
    if (leader) r = wait_bar<SW>(bar, parity, abort_flag, a.status) ? 1 : 0;
    return __shfl_sync(0xffffffffu, r, 0) != 0;
  };
  // gathered tile: lanes' copies, then the barrier takes them over
  auto gather_into = [&](unsigned char* dst, const void* src, int m0, uint64_t* bar) {
    gather_rows<D>(dst, static_cast<const __nv_bfloat16*>(src), m0, N, F, P);
    cp_async_mbar_arrive(bar);
    __syncwarp();
    if (leader) mbar_arrive(bar);
  };
  // Ring entry l is free (its previous occupant released).  With one MMA
  // issuer the K and V entries of a step are claimed one at a time: a K tile
  // is released after the two Q K^T of its step, a V tile only after the two
  // P.V, which that thread issues while serving the next step, so the next K
  // load does not wait for the last P.V.  With an issuer per member both
  // entries are claimed before the K copy: a member that skips a step
  // releases the step's V entry at once, and were the next K tile loaded
  // first it could pass the reuse of that entry and release it a second
  // time before the other member's P.V has read it.
  auto claim = [&](uint32_t l) -> bool {
    return leader_wait(&B.kv_empty[l % S], ((l / S) & 1) ^ 1);
  };
  // claims made before the copy of entry L + kv of a step
  auto claim_step = [&](int kv) -> bool {
    if (C::kOneIssuer) return claim(L + kv);
    return kv == 1 || (claim(L) && claim(L + 1));
  };
  uint32_t issued = 0;  // ring entries whose copies were issued
  for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
    const int bh = item / n_pairs, qt0 = 2 * (item - bh * n_pairs);
    const bool tm = gathers_input(a, bh);
    const bool cp = reads_copies(a, bh);
    const uint32_t vexp = v_exponent(a, bh);
    const CUtensorMap* mq = cp ? &maps.qt : &maps.q;
    const CUtensorMap* mk = cp ? &maps.kt : &maps.k;
    const CUtensorMap* mv = cp ? &maps.vt : &maps.v;
    const long long head = static_cast<long long>(bh) * N * D;
    int p[2], e[2], qtile[2];
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      qtile[t] = query_tile(a, bh, qt0 + t, nb);
      if (qtile[t] < 0 && qt0 + t < nb && leader) set_status(a.status, SVG_DEVICE_BAD_INDEX);
      member_list(a, bh, qtile[t], nb, p[t], e[t], leader);
      skip_invalid(a, nb, p[t], e[t], -1, leader);
    }
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      if (p[t] >= e[t] || !ok) continue;
      const uint32_t qs = cq[t] % QD, qb = t * QD + qs;
      if (!(ok = leader_wait(&B.q_empty[qb], ((cq[t] / QD) & 1) ^ 1))) continue;
      unsigned char* dst = smem + C::kOffQ + qb * C::kTile;
      if (!tm) {
        if (leader) {
          mbar_arrive_expect_tx(&B.q_full[qb], C::kTile);
          for (int bx = 0; bx < C::kBoxes; ++bx)
            tma_load_3d(dst + bx * kBox, mq, &B.q_full[qb], 64 * bx, qtile[t] * 128, bh);
        }
      } else {
        gather_into(dst, static_cast<const __nv_bfloat16*>(a.q) + head, qtile[t] * 128,
                    &B.q_full[qb]);
      }
      ++cq[t];
    }
    uint32_t seen = 0;  // members that already had a block in this item
    int j, mask;
    while (ok && merge_next(a, nb, p, e, j, mask, leader)) {
      const uint32_t m = static_cast<uint32_t>(mask);
      const uint32_t last = (m & 1u) * (p[0] >= e[0] ? 1u : 0u) |
                            (m & 2u) * (p[1] >= e[1] ? 1u : 0u);
      const uint32_t info = m | ((m & ~seen) << 2) | (last << 4) | (tm ? kStepGathered : 0u) |
                            (vexp << kStepExpShift);
      seen |= m;
      for (int kv = 0; kv < 2; ++kv) {
        if (!(ok = claim_step(kv))) break;
        // the record is read after the step's K entry is full
        if (kv == 0 && leader) step_info[(L / 2) % C::kInfo] = info;
        const uint32_t slot = (L + kv) % S;
        unsigned char* dst = smem + C::kOffKV + slot * C::kTile;
        const void* src = kv == 0 ? a.k : a.v;
        if (!tm) {
          if (leader) {
            mbar_arrive_expect_tx(&B.kv_full[slot], C::kTile);
            const CUtensorMap* map = kv == 0 ? mk : mv;
            for (int bx = 0; bx < C::kBoxes; ++bx)
              tma_load_3d(dst + bx * kBox, map, &B.kv_full[slot], 64 * bx, j * 128, bh);
          }
        } else {
          gather_into(dst, static_cast<const __nv_bfloat16*>(src) + head, j * 128,
                      &B.kv_full[slot]);
        }
        issued = L + kv + 1;
      }
      L += 2;
    }
  }
  // end record in the next step's entries; plain arrives complete their
  // phases
  for (int kv = 0; kv < 2 && ok; ++kv) {
    if (!(ok = claim_step(kv))) break;
    if (leader) {
      if (kv == 0) step_info[(L / 2) % C::kInfo] = kStepEnd;
      mbar_arrive(&B.kv_full[(L + kv) % S]);
    }
  }
  if (!ok) {
    // let the copies already issued land before the CTA can exit
    cp_async_wait<0>();
    if (leader) {
      for (uint32_t l = issued > S ? issued - S : 0; l < issued; ++l)
        drain_bar(&B.kv_full[l % S], (l / S) & 1);
      for (int t = 0; t < 2; ++t)
        for (uint32_t c = cq[t] > QD ? cq[t] - QD : 0; c < cq[t]; ++c)
          drain_bar(&B.q_full[t * QD + c % QD], (c / QD) & 1);
    }
  }
}

// MMA issuer (one thread).  With kOneIssuer it serves both members in a
// fixed order per step: member 0's pending P.V, member 0's Q K^T, member 1's
// pending P.V, member 1's Q K^T.  The tensor core runs its instructions in
// issue order, so member 1's scores land one P.V + Q K^T after member 0's and
// the two softmax warpgroups take turns on the exponential unit instead of
// sharing it.  (Without kOneIssuer each member has an issuer thread of its
// own, issuer_member.)  The thread serves members t0 .. t1.
template <int D, int t0, int t1, bool SW>
__device__ __forceinline__ void issuer(const Bars& B, unsigned char* smem,
                                       volatile uint32_t* step_info, volatile int* abort_flag,
                                       uint32_t tmem, int32_t* status) {
  using C = Cfg<D>;
  constexpr int QD = C::kQDepth, S = C::kSlots;
  uint32_t t_s[2], t_p[2], t_o[2];
  uint64_t dq[2];
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    t_s[t] = tmem + C::kColS + 128 * t;
    t_p[t] = tmem + C::kColP + C::kPStride * t;
    t_o[t] = tmem + C::kColO + C::kOStride * t;
    // descriptor of the member's first Q buffer; a buffer at byte offset x
    // adds x >> 4 (the start-address field)
    dq[t] = sdesc_sw128(smem_u32(smem + C::kOffQ + t * QD * C::kTile), 16, 1024);
  }
  const uint64_t dk = sdesc_sw128(smem_u32(smem + C::kOffKV), 16, 1024);
  const uint64_t dv = sdesc_sw128(smem_u32(smem + C::kOffKV), kBox, 1024);
  uint32_t L = 0, cq[2] = {0, 0}, nq[2] = {0, 0}, np[2] = {0, 0}, pend_lv[2] = {0, 0};
  bool ok = true, pend[2] = {false, false}, pend_first[2] = {false, false};
  auto issue_pv = [&](int t) -> bool {
    if (!wait_bar<SW>(&B.p_ready[t], np[t] & 1, abort_flag, status)) return false;
    const uint32_t slot = pend_lv[t] % S;
    if (!wait_bar<SW>(&B.v_ready[slot], (pend_lv[t] / S) & 1, abort_flag, status)) return false;
    tc_fence_after();
    const uint64_t d0 = dv + ((slot * C::kTile) >> 4);
    mma_ts_k128(t_o[t], t_p[t], d0, C::kIdescPV, pend_first[t] ? 0u : 1u);
    tc_commit(&B.o_done[t]);
    tc_commit(&B.kv_empty[slot]);
    ++np[t];
    pend[t] = false;
    return true;
  };
  while (ok) {
    const uint32_t kslot = L % S;
    if (!(ok = wait_bar<SW>(&B.kv_full[kslot], (L / S) & 1, abort_flag, status))) break;
    const uint32_t info = step_info[(L / 2) % C::kInfo];
    // gathered tiles were written through the generic proxy
    if (info & kStepGathered) fence_proxy_async_smem();
    if (info & kStepEnd) break;
#pragma unroll
    for (int t = 0; t < 2; ++t) {  // unrolled: the per-member state stays in registers
      if (t < t0 || t > t1 || !ok) continue;
      if (!(info >> t & 1u)) {
        // this member skips the block: its pending P.V goes now (otherwise
        // that V entry could stay held past the point where the producer
        // needs it again), then its share of both entries is released
        if (pend[t] && !(ok = issue_pv(t))) continue;
        tc_commit(&B.kv_empty[kslot]);
        tc_commit(&B.kv_empty[kslot + 1]);
        continue;
      }
      if constexpr (!C::kSepP) {
        // P_t lives in S_t: the previous P.V goes first (tensor-core order)
        if (pend[t] && !(ok = issue_pv(t))) continue;
      } else if (nq[t] > 0) {
        if (!(ok = wait_bar<SW>(&B.s_free[t], (nq[t] - 1) & 1, abort_flag, status))) continue;
      }
      const uint32_t qs = cq[t] % QD;
      if (info >> (2 + t) & 1u) {  // first block of the item: a new Q tile
        if (!(ok = wait_bar<SW>(&B.q_full[t * QD + qs], (cq[t] / QD) & 1, abort_flag, status)))
          continue;
        if (info & kStepGathered) fence_proxy_async_smem();
      }
      tc_fence_after();
      const uint64_t q0 = dq[t] + ((qs * C::kTile) >> 4), k0 = dk + ((kslot * C::kTile) >> 4);
      if constexpr (D == 64)
        mma_ss_k64(t_s[t], q0, k0, C::kIdescQK);
      else
        mma_ss_k128(t_s[t], q0, k0, C::kIdescQK, kBox >> 4);
      tc_commit(&B.s_full[t]);
      tc_commit(&B.kv_empty[kslot]);
      if (info >> (4 + t) & 1u) {  // last block of the item: its Q buffer is free
        tc_commit(&B.q_empty[t * QD + qs]);
        ++cq[t];
      }
      ++nq[t];
      if constexpr (C::kSepP) {
        if (pend[t] && !(ok = issue_pv(t))) continue;
      }
      pend[t] = true;
      pend_first[t] = (info >> (2 + t)) & 1u;
      pend_lv[t] = L + 1;
    }
    L += 2;
  }
#pragma unroll
  for (int t = 0; t < 2; ++t)
    if (t >= t0 && t <= t1 && ok && pend[t]) ok = issue_pv(t);
  // every MMA issued by this thread completes before TMEM is released
  tc_commit(&B.drain[t0]);
  drain_bar(&B.drain[t0], 0);
}

// MMA issuer of one member (two-issuer mode): the same steps as `issuer`
// for member t alone.  One copy of this code serves both issuer warps (t is a
// runtime value), which keeps the kernel's instruction footprint small.
template <int D, bool SW>
__device__ __forceinline__ void issuer_member(const Bars& B, unsigned char* smem,
                                              volatile uint32_t* step_info,
                                              volatile int* abort_flag, uint32_t tmem,
                                              int32_t* status, int t) {
  using C = Cfg<D>;
  constexpr int QD = C::kQDepth, S = C::kSlots;
  const uint32_t t_s = tmem + C::kColS + 128 * t;
  const uint32_t t_p = tmem + C::kColP + C::kPStride * t;
  const uint32_t t_o = tmem + C::kColO + C::kOStride * t;
  // descriptors of the member's first Q buffer and of ring entry 0; a buffer
  // at byte offset x adds x >> 4 (the start-address field)
  const uint64_t dq = sdesc_sw128(smem_u32(smem + C::kOffQ + t * QD * C::kTile), 16, 1024);
  const uint64_t dk = sdesc_sw128(smem_u32(smem + C::kOffKV), 16, 1024);
  const uint64_t dv = sdesc_sw128(smem_u32(smem + C::kOffKV), kBox, 1024);
  uint32_t L = 0, cq = 0, nq = 0, np = 0, pend_lv = 0;
  bool ok = true, pend = false, pend_first = false;
  auto issue_pv = [&]() -> bool {
    if (!wait_bar<SW>(&B.p_ready[t], np & 1, abort_flag, status)) return false;
    const uint32_t slot = pend_lv % S;
    if (!wait_bar<SW>(&B.v_ready[slot], (pend_lv / S) & 1, abort_flag, status)) return false;
    tc_fence_after();
    mma_ts_k128(t_o, t_p, dv + ((slot * C::kTile) >> 4), C::kIdescPV, pend_first ? 0u : 1u);
    tc_commit(&B.o_done[t]);
    tc_commit(&B.kv_empty[slot]);
    ++np;
    pend = false;
    return true;
  };
  while (ok) {
    const uint32_t kslot = L % S;
    if (!(ok = wait_bar<SW>(&B.kv_full[kslot], (L / S) & 1, abort_flag, status))) break;
    const uint32_t info = step_info[(L / 2) % C::kInfo];
    if (info & kStepGathered) fence_proxy_async_smem();
    if (info & kStepEnd) break;
    if (!(info >> t & 1u)) {  // skipped block: as in `issuer`
      if (pend && !(ok = issue_pv())) break;
      tc_commit(&B.kv_empty[kslot]);
      tc_commit(&B.kv_empty[kslot + 1]);
      L += 2;
      continue;
    }
    if constexpr (!C::kSepP) {
      if (pend && !(ok = issue_pv())) break;
    } else if (nq > 0) {
      if (!(ok = wait_bar<SW>(&B.s_free[t], (nq - 1) & 1, abort_flag, status))) break;
    }
    const uint32_t qs = cq % QD;
    if (info >> (2 + t) & 1u) {
      if (!(ok = wait_bar<SW>(&B.q_full[t * QD + qs], (cq / QD) & 1, abort_flag, status))) break;
      if (info & kStepGathered) fence_proxy_async_smem();
    }
    tc_fence_after();
    const uint64_t q0 = dq + ((qs * C::kTile) >> 4), k0 = dk + ((kslot * C::kTile) >> 4);
    if constexpr (D == 64)
      mma_ss_k64(t_s, q0, k0, C::kIdescQK);
    else
      mma_ss_k128(t_s, q0, k0, C::kIdescQK, kBox >> 4);
    tc_commit(&B.s_full[t]);
    tc_commit(&B.kv_empty[kslot]);
    if (info >> (4 + t) & 1u) {
      tc_commit(&B.q_empty[t * QD + qs]);
      ++cq;
    }
    ++nq;
    if constexpr (C::kSepP) {
      if (pend && !(ok = issue_pv())) break;
    }
    pend = true;
    pend_first = (info >> (2 + t)) & 1u;
    pend_lv = L + 1;
    L += 2;
  }
  if (ok && pend) ok = issue_pv();
  tc_commit(&B.drain[t]);
  drain_bar(&B.drain[t], 0);
}

// Converts every V tile in place from bf16 to fp16, in ring order; `part` of
// C::kConvWarps warps (each takes every kConvWarps-th 16-byte piece, and
// each arrives once on the tile's v_ready).  bf16 -> fp16 is exact for
// |v| <= 65504 (fp16 subnormals keep the absolute error below 2^-25);
// larger values become inf and are reported as SVG_DEVICE_RANGE.  The check
// is on the bf16 bits: a magnitude field of 0x4780 (65536) or more, inf and
// NaN included, carries into bit 15 of its half once 0x3880 is added, and the
// 15-bit fields cannot carry into each other.
template <int D, bool SW>
__device__ __forceinline__ void converter(const AttnArgs& a, const Bars& B, unsigned char* smem,
                                          volatile uint32_t* step_info, volatile int* abort_flag,
                                          int part) {
  using C = Cfg<D>;
  constexpr int S = C::kSlots;
  const int lane = threadIdx.x & 31;
  uint32_t L = 0, over = 0;
  bool ok = true;
  while (ok) {
    const uint32_t slot = (L + 1) % S;
    if (!(ok = wait_bar<SW>(&B.kv_full[slot], ((L + 1) / S) & 1, abort_flag, a.status))) break;
    const uint32_t info = step_info[(L / 2) % C::kInfo];
    if (info & kStepEnd) break;
    uint4* tile = reinterpret_cast<uint4*>(smem + C::kOffKV + slot * C::kTile);
    const uint32_t e = (info >> kStepExpShift) & 0xffu;
    if (e == 0) {
#pragma unroll 4
      for (int c = part * 32 + lane; c < C::kTile / 16; c += 32 * C::kConvWarps) {
        uint4 v = tile[c];
        uint32_t* w = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float lo = __uint_as_float(w[i] << 16), hi = __uint_as_float(w[i] & 0xffff0000u);
          over |= (w[i] & 0x7fff7fffu) + 0x38803880u;
          const __half2 h = __floats2half2_rn(lo, hi);
          w[i] = *reinterpret_cast<const uint32_t*>(&h);
        }
        tile[c] = v;
      }
    } else {
      // v * 2^-e (exact), which the head's exponent brings into fp16 range
      const float sc = __uint_as_float((127u - e) << 23);
#pragma unroll 4
      for (int c = part * 32 + lane; c < C::kTile / 16; c += 32 * C::kConvWarps) {
        uint4 v = tile[c];
        uint32_t* w = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const __half2 h = __floats2half2_rn(__uint_as_float(w[i] << 16) * sc,
                                              __uint_as_float(w[i] & 0xffff0000u) * sc);
          w[i] = *reinterpret_cast<const uint32_t*>(&h);
        }
        tile[c] = v;
      }
    }
    fence_proxy_async_smem();  // generic-proxy writes -> tensor-core reads
    __syncwarp();
    if (lane == 0) mbar_arrive(&B.v_ready[slot]);
    L += 2;
  }
  if (__any_sync(0xffffffffu, (over & 0x80008000u) != 0u) && lane == 0)
    set_status(a.status, SVG_DEVICE_RANGE);
}

template <int D, bool SW>
__global__ void __launch_bounds__(kThreads, 1)
    attn_sm100_kernel(const __grid_constant__ Maps maps, const AttnArgs a) {
  using C = Cfg<D>;
  constexpr int QD = C::kQDepth, S = C::kSlots;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bar_base = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  Bars B;
  B.q_full = bar_base;
  B.q_empty = B.q_full + 2 * QD;
  B.kv_full = B.q_empty + 2 * QD;
  B.kv_empty = B.kv_full + S;
  B.v_ready = B.kv_empty + S;
  B.s_full = B.v_ready + S;
  B.s_free = B.s_full + 2;
  B.p_ready = B.s_free + 2;
  B.o_done = B.p_ready + 2;
  B.drain = B.o_done + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(B.drain + 2);
  // abort flag, then the poll limit of every wait
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile uint32_t* step_info = reinterpret_cast<volatile uint32_t*>(smem + C::kOffInfo);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int N = a.N, nb = n_tiles(N);
  const int n_pairs = (nb + 1) / 2;
  const int n_items = a.B * a.H * n_pairs;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2 * QD; ++i) {
      mbar_init(&B.q_full[i], 1);
      mbar_init(&B.q_empty[i], 1);
    }
    for (int i = 0; i < S; ++i) {
      mbar_init(&B.kv_full[i], 1);
      mbar_init(&B.kv_empty[i], 2);
      mbar_init(&B.v_ready[i], C::kConvWarps);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&B.s_full[t], 1);
      mbar_init(&B.s_free[t], 4);
      mbar_init(&B.p_ready[t], 4);
      mbar_init(&B.o_done[t], 1);
      mbar_init(&B.drain[t], 1);
    }
    abort_flag[0] = 0;
    abort_flag[1] = static_cast<int>(min(a.spin_limit, 0x7fffffffu));
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&maps.q);
    prefetch_tmap(&maps.k);
    prefetch_tmap(&maps.v);
    if (a.q_tm != nullptr) {
      prefetch_tmap(&maps.qt);
      prefetch_tmap(&maps.kt);
      prefetch_tmap(&maps.vt);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    reg_dealloc<C::kRegsLow>();
    // ------------------------------------------------------------ producer
    producer<D, SW>(a, maps, B, smem, step_info, abort_flag, n_items, n_pairs, nb);
  } else if (warp == 1 || (warp == 2 && !C::kOneIssuer)) {
    reg_dealloc<C::kRegsLow>();
    // ------------------------------------------------------------ MMA issuers
    if (lane == 0) {
      if constexpr (C::kOneIssuer)
        issuer<D, 0, 1, SW>(B, smem, step_info, abort_flag, tmem, a.status);
      else
        issuer_member<D, SW>(B, smem, step_info, abort_flag, tmem, a.status, warp - 1);
    }
  } else if (warp <= 3) {
    reg_dealloc<C::kRegsLow>();
    // ------------------------------------------------------------ V to fp16
    // (the converter warps are the last kConvWarps of warpgroup 0)
    if (warp >= 4 - C::kConvWarps)
      converter<D, SW>(a, B, smem, step_info, abort_flag, warp - (4 - C::kConvWarps));
  } else {
    reg_alloc<C::kRegsHigh>();
    softmax_member<D, SW>(a, B, abort_flag, tmem, n_items, n_pairs, nb);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------ host side

}  // namespace

template <int D>
svg_status launch_attn_sm100(const AttnArgs& a, cudaStream_t s) {
  using C = Cfg<D>;
  Maps maps = {};
  const int BH = a.B * a.H;
  if (!make_tma_map_3d(&maps.q, a.q, BH, a.N, D) || !make_tma_map_3d(&maps.k, a.k, BH, a.N, D) ||
      !make_tma_map_3d(&maps.v, a.v, BH, a.N, D) ||
      (a.q_tm != nullptr && (!make_tma_map_3d(&maps.qt, a.q_tm, BH, a.N, D) ||
                             !make_tma_map_3d(&maps.kt, a.k_tm, BH, a.N, D) ||
                             !make_tma_map_3d(&maps.vt, a.v_tm, BH, a.N, D))))
    return fail(SVG_ERR_CUDA, "sparse_attn: cannot encode TMA descriptors");
  // a launch with a poll limit other than the default runs the instantiation
  // that reads it (the same code otherwise)
  const bool sw = a.spin_limit != kDefaultWaitLimit;
  auto kernel = sw ? attn_sm100_kernel<D, true> : attn_sm100_kernel<D, false>;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem) !=
      cudaSuccess)
    return fail(SVG_ERR_CUDA, "sparse_attn: cannot reserve %d bytes of shared memory", C::kSmem);
  const long long items = static_cast<long long>(BH) * ((n_tiles(a.N) + 1) / 2);
  const int grid = static_cast<int>(items < sm_count() ? items : sm_count());
  kernel<<<grid, kThreads, C::kSmem, s>>>(maps, a);
  return check_launch("sparse_attn sm100");
}

template svg_status launch_attn_sm100<64>(const AttnArgs&, cudaStream_t);
template svg_status launch_attn_sm100<128>(const AttnArgs&, cudaStream_t);

}  // namespace svg
