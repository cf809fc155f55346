// Online head profiling.
//
// Sparse VideoGen article (m.jxzklqfsx.com/article/815093.html), section
// "動態自適應的稀疏策略", steps 1-3: at every step a few query tokens (about
// 64) are sampled; their attention outputs are computed under the spatial and
// the temporal mask and compared with dense attention; each head takes the
// mask with the smaller error.  Error = mean over the S x d sampled outputs of
// the squared difference; an exact tie keeps SPATIAL.
//
// Work split (one layer, all heads, one launch each):
//   partial  the keys of a head are cut into `chunks` contiguous ranges (a
//            multiple of 128 keys each); a unit is one (range, head).  bf16:
//            a persistent tcgen05 kernel, one CTA per SM looping over units,
//            the 64 sampled rows as one M = 128 tile, K and V streamed by TMA
//            through rings of their own, S = Q K^T and both P.V products on
//            the tensor core with TMEM accumulators, and two online-softmax
//            states per row (dense, and under the spatial mask: each row's
//            band of frames is one contiguous key range, tested with two
//            compares) sharing one Q K^T per tile.  fp32: SIMT, one launch
//            per mask (grid z).
//   merge    grid (B*H, 16), one warp per sampled row: the chunk weights
//            exp2(m_c - M) / L, the merged dense and spatial outputs, the
//            temporal output (a row sees only the F keys of its position,
//            computed directly) and the row's squared errors;
//   finalize grid (B*H): mean errors and the mode.
// The pass reads K and V once per head and costs a few percent of the
// attention it configures.
#include <float.h>
#include <limits.h>

#include "common.cuh"
#include "sm100.cuh"

namespace svg {
namespace {

constexpr int kRows = 64;          // sampled rows per head (S padded to 64)
constexpr int kTileKeys = 128;     // keys per tile of the tcgen05 path; ranges are multiples
constexpr int kSms = 148;          // persistent CTAs the chunking plans for (B200)
constexpr int kUnitTiles = 2;      // fixed cost of a unit (Q gather, fill, epilogue) in tiles
constexpr int kMaxChunks = 32;     // merge holds one chunk weight per lane
constexpr float kLog2e = 1.4426950408889634f;

// Sampled indices outside [0, N) are clamped into range (never read out of bounds).
__device__ __forceinline__ int clamp_index(int n, int N) { return n < 0 ? 0 : (n >= N ? N - 1 : n); }

struct ProfileShape {
  int chunks;     // key ranges per head
  int chunk_len;  // keys per range (multiple of kTileKeys)
};

ProfileShape shape_for(int N, long long chunks) {
  const long long max_chunks = (N + 4 * kTileKeys - 1) / (4 * kTileKeys);  // >= 4 tiles per range
  if (chunks > max_chunks) chunks = max_chunks;
  if (chunks > kMaxChunks) chunks = kMaxChunks;
  if (chunks < 1) chunks = 1;
  long long len = (N + chunks - 1) / chunks;
  len = (len + kTileKeys - 1) / kTileKeys * kTileKeys;
  chunks = (N + len - 1) / len;
  return {static_cast<int>(chunks), static_cast<int>(len)};
}

// The key-range count whose busiest CTA does the least: units of one
// (range, head) go round-robin to kSms persistent CTAs, so the critical path
// is ceil(units / kSms) units of (tiles per range + kUnitTiles) tiles each.
// Ties go to fewer ranges (less merge work).
ProfileShape profile_shape(int B, int H, int N) {
  const long long bh = static_cast<long long>(B) * H;
  ProfileShape best = shape_for(N, 1);
  long long best_cost = -1;
  for (int c = 1; c <= kMaxChunks; ++c) {
    const ProfileShape ps = shape_for(N, c);
    const long long rounds = (bh * ps.chunks + kSms - 1) / kSms;
    const long long cost = rounds * (ps.chunk_len / kTileKeys + kUnitTiles);
    if (best_cost < 0 || cost < best_cost) {
      best = ps;
      best_cost = cost;
    }
  }
  return best;
}

// floats per partial state row: m, l, o[D]
template <int D>
constexpr int state_floats() {
  return D + 2;
}

size_t states_bytes(int B, int H, int chunks, int d) {
  const size_t b = static_cast<size_t>(B) * H * 2 * chunks * kRows * (d + 2) * sizeof(float);
  return (b + 255) / 256 * 256;
}

// per (head, sampled row): squared errors of the spatial and temporal outputs
size_t errors_bytes(int B, int H) {
  return (static_cast<size_t>(B) * H * kRows * 2 * sizeof(float) + 255) / 256 * 256;
}

size_t partial_bytes(int B, int H, int N, int d) {
  ProfileShape ps = profile_shape(B, H, N);
  return states_bytes(B, H, ps.chunks, d) + errors_bytes(B, H);
}

// --------------------------------------------------------------- fp32 partial

// SIMT fp32: warp per sampled row, lanes split the head dimension; grid z
// selects the mask (0 dense, 1 spatial).
template <int D>
__global__ void __launch_bounds__(256) profile_partial_fp32(
    const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
    const int32_t* __restrict__ idx, int S, int N, int P, int width, float scale_log2, int chunks,
    int chunk_len, float* __restrict__ ws) {
  constexpr int E = D / 32;
  const int chunk = blockIdx.x, bh = blockIdx.y, variant = blockIdx.z;
  const long long head = static_cast<long long>(bh) * N * D;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int key_begin = chunk * chunk_len;
  const int key_end = min(N, key_begin + chunk_len);
  float* base = ws + ((static_cast<long long>(bh) * 2 + variant) * chunks + chunk) * kRows *
                         state_floats<D>();
  for (int r = warp; r < kRows; r += 8) {
    float m = -INFINITY, l = 0.f, acc[E], qv[E];
    const int n = r < S ? clamp_index(idx[r], N) : 0;
    const int fr = n / P;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      acc[e] = 0.f;
      qv[e] = r < S ? q[head + static_cast<long long>(n) * D + lane + 32 * e] : 0.f;
    }
    if (r < S) {
      for (int j = key_begin; j < key_end; ++j) {
        if (variant == 1 && abs(j / P - fr) > width) continue;
        float dot = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e)
          dot = fmaf(qv[e], k[head + static_cast<long long>(j) * D + lane + 32 * e], dot);
#pragma unroll
        for (int o2 = 16; o2 > 0; o2 >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o2);
        const float t = dot * scale_log2;
        const float mn = fmaxf(m, t);
        const float alpha = exp2f(m - mn);
        const float p = exp2f(t - mn);
        l = l * alpha + p;
#pragma unroll
        for (int e = 0; e < E; ++e)
          acc[e] = fmaf(p, v[head + static_cast<long long>(j) * D + lane + 32 * e], acc[e] * alpha);
        m = mn;
      }
    }
    float* row = base + r * state_floats<D>();
    if (lane == 0) {
      row[0] = m;
      row[1] = l;
    }
#pragma unroll
    for (int e = 0; e < E; ++e) row[2 + lane + 32 * e] = acc[e];
  }
}

// --------------------------------------------------------------- tcgen05 partial (bf16)
//
// Persistent, one CTA per SM, looping over work units (key range c, head bh).
// The M = 128 tile holds the 64 sampled rows twice: rows 0-63 for the dense
// state, rows 64-127 (the same queries) for the state under the spatial mask.
// One Q K^T gives both copies of the scores, and one P.V (P of the dense
// state in TMEM lanes 0-63, of the spatial state in lanes 64-127) gives both
// outputs.  Seven warps:
//   warps 0-3   softmax: warp w owns TMEM lanes 32 w .. 32 w + 31, i.e.
//               sampled rows 32 (w & 1) + lane of state w >> 1 (0 dense,
//               1 spatial), and works through every 128-key tile of the unit
//               for them (fp32 online softmax with lazy rescaling: an output
//               is rescaled only when its running max grows by more than 2^8;
//               the weights go to TMEM as bf16 over the scores they came
//               from, and the row sums add the same rounded values).  A
//               spatial warp whose rows have no band key in a tile writes
//               zero weights without touching the scores;
//   warp 4      K loader: gathers the unit's sampled Q rows (cp.async, into
//               both halves of the 128-byte-swizzled K-major Q tile), then
//               streams the K tiles of the range through a ring (TMA);
//   warp 5      MMA issuer (one thread): S_j = Q K_j^T into one of two TMEM
//               score buffers, then O += P_j-1 V_j-1 with P from TMEM and V
//               from shared memory;
//   warp 6      V loader: the V tiles through a ring of their own, so that a
//               K entry is refilled as soon as its Q K^T is done while a V
//               entry waits for its P.V.
// The scores of tile j are computed while the softmax works on tile j-1.
// Every wait is bounded; a CTA that gives up writes NaN into the states of
// its units (so the head's errors come out NaN) and drains.

constexpr int kTcThreads = 224;

template <int D>
struct TcCfg {
  static constexpr int kTile = 128 * D * 2;         // a 128-row Q / K / V tile
  static constexpr int kBox = 16384;                // 128 rows x 128 bytes
  static constexpr int kBoxes = D / 64;
  static constexpr int kStages = D == 64 ? 6 : 3;   // K ring and V ring entries each
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kTile;               // [stage]
  static constexpr int kOffV = kOffK + kStages * kTile;
  static constexpr int kOffBar = kOffV + kStages * kTile;
  // q_full, q_empty, k_full[S], k_empty[S], v_full[S], v_empty[S], s_full[2],
  // p_ready[2], o_done, drain
  static constexpr int kBars = 2 + 4 * kStages + 2 + 2 + 2;
  static constexpr int kSmem = kOffBar + kBars * 8 + 16 + 1024;  // + the base's 1024-byte alignment
  static constexpr uint32_t kColS = 0;  // S_b at 128 b; P_b (bf16) over its columns 0-63
  static constexpr uint32_t kColO = 256;
  static constexpr uint32_t kIdescQK = sm100::idesc_bf16(128, 128, false);
  static constexpr uint32_t kIdescPV = sm100::idesc_bf16(128, D, true);
  static_assert(kSmem <= 227 * 1024, "shared memory budget");
};

constexpr uint32_t kTcSpin = 1u << 22;
constexpr uint32_t kTcDrain = 1u << 20;
constexpr unsigned kNapIssue = 32;   // ns between polls of the MMA issuer
constexpr unsigned kNapLoad = 128;   // ns between polls of the loaders

__device__ __forceinline__ bool tc_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  const uint32_t addr = smem_u32(bar);
  for (uint32_t i = 0; i < kTcSpin; ++i) {
    if (sm100::mbar_try_wait(addr, parity)) return true;
    if ((i & 255u) == 255u && *abort_flag) return false;
  }
  *abort_flag = 1;
  return false;
}
// The helper warps (loaders, issuer) share their SM sub-partitions with the
// softmax warps: between polls they sleep for `ns` nanoseconds instead of
// taking issue slots.  Bounded like tc_wait.
__device__ __forceinline__ bool tc_wait_nap(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                            unsigned ns) {
  const uint32_t addr = smem_u32(bar);
  for (uint32_t i = 0; i < kTcSpin; ++i) {
    if (sm100::mbar_try_wait(addr, parity)) return true;
    if ((i & 255u) == 255u && *abort_flag) return false;
    __nanosleep(ns);
  }
  *abort_flag = 1;
  return false;
}
// The same wait taken by a whole warp: every lane leaves with the same answer,
// so a timeout cannot split the warp across the warp-wide instructions after it.
__device__ __forceinline__ bool tc_wait_warp(uint64_t* bar, uint32_t parity,
                                             volatile int* abort_flag) {
  return __all_sync(0xffffffffu, tc_wait(bar, parity, abort_flag)) != 0;
}
__device__ __forceinline__ void tc_drain(uint64_t* bar, uint32_t parity) {
  const uint32_t addr = smem_u32(bar);
  for (uint32_t i = 0; i < kTcDrain; ++i)
    if (sm100::mbar_try_wait(addr, parity)) return;
}

struct TcUnit {
  int bh, chunk, key_begin, key_end, tiles;
};
__device__ __forceinline__ TcUnit tc_unit(int u, int chunks, int chunk_len, int N) {
  TcUnit w;
  w.bh = u / chunks;
  w.chunk = u - w.bh * chunks;
  w.key_begin = w.chunk * chunk_len;
  w.key_end = min(N, w.key_begin + chunk_len);
  w.tiles = w.key_end > w.key_begin ? (w.key_end - w.key_begin + kTileKeys - 1) / kTileKeys : 0;
  return w;
}

// The state row [m, l, o[D]] of sampled row r, variant (0 dense, 1 spatial),
// of unit w in the workspace [bh][variant][chunk][row].
template <int D>
__device__ __forceinline__ float* tc_state_row(float* ws, const TcUnit& w, int variant, int r,
                                               int chunks) {
  return ws + ((static_cast<long long>(w.bh) * 2 + variant) * chunks + w.chunk) * kRows *
                  state_floats<D>() +
         static_cast<long long>(r) * state_floats<D>();
}

template <int D>
__global__ void __launch_bounds__(kTcThreads, 1) profile_partial_tc(
    const __grid_constant__ CUtensorMap mk, const __grid_constant__ CUtensorMap mv,
    const __nv_bfloat16* __restrict__ q, const int32_t* __restrict__ idx, int S, int N, int P,
    int width, float scale_log2, int chunks, int chunk_len, int n_units,
    float* __restrict__ ws) {
  using C = TcCfg<D>;
  using namespace sm100;
  constexpr int ST = C::kStages;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* q_full = bars;
  uint64_t* q_empty = bars + 1;
  uint64_t* k_full = bars + 2;
  uint64_t* k_empty = k_full + ST;
  uint64_t* v_full = k_empty + ST;
  uint64_t* v_empty = v_full + ST;
  uint64_t* s_full = v_empty + ST;
  uint64_t* p_ready = s_full + 2;
  uint64_t* o_done = p_ready + 2;
  uint64_t* drain = o_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < ST; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&p_ready[b], 4);
    }
    mbar_init(o_done, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ------------------------------------------------------------------ K loader
    if (lane == 0) {
      prefetch_tmap(&mk);
      prefetch_tmap(&mv);
    }
    constexpr int CH = D / 8;  // 16-byte chunks per row
    uint32_t gt = 0, nu = 0;  // tiles and units loaded
    bool ok = true;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
      const TcUnit w = tc_unit(u, chunks, chunk_len, N);
      if (w.tiles == 0) continue;
      int r_ok = 1;
      if (lane == 0) r_ok = tc_wait_nap(q_empty, (nu & 1) ^ 1, abort_flag, kNapLoad) ? 1 : 0;
      if (!(ok = __shfl_sync(0xffffffffu, r_ok, 0) != 0)) break;
      ++nu;
      // sampled row r into tile rows r and r + 64 (same swizzle phase: r & 7)
      const __nv_bfloat16* qh = q + static_cast<long long>(w.bh) * N * D;
      for (int t = lane; t < kRows * CH; t += 32) {
        const int r = t / CH, c = t % CH;
        const bool valid = r < S;
        const int n = valid ? clamp_index(idx[r], N) : 0;
        const __nv_bfloat16* src = qh + static_cast<long long>(n) * D + c * 8;
        unsigned char* dst = smem + C::kOffQ + (c >> 3) * C::kBox + r * 128 + (((c & 7) ^ (r & 7)) << 4);
        cp_async16(dst, src, valid);
        cp_async16(dst + kRows * 128, src, valid);
      }
      cp_async_mbar_arrive(q_full);
      __syncwarp();
      if (lane == 0) mbar_arrive(q_full);
      for (int j = 0; j < w.tiles; ++j) {
        const uint32_t st = gt % ST;
        int r_ok = 1;  // lane 0 waits and copies; the warp learns the outcome
        if (lane == 0) {
          if (tc_wait_nap(&k_empty[st], ((gt / ST) & 1) ^ 1, abort_flag, kNapLoad)) {
            mbar_arrive_expect_tx(&k_full[st], C::kTile);
            const int key0 = w.key_begin + j * kTileKeys;
            for (int bx = 0; bx < C::kBoxes; ++bx)
              tma_load_3d(smem + C::kOffK + st * C::kTile + bx * C::kBox, &mk, &k_full[st],
                          64 * bx, key0, w.bh);
          } else {
            r_ok = 0;
          }
        }
        if (!(ok = __shfl_sync(0xffffffffu, r_ok, 0) != 0)) break;
        ++gt;
      }
    }
    cp_async_wait<0>();
    if (!ok && lane == 0) {  // copies in flight land before the CTA can exit
      for (uint32_t l = gt > ST ? gt - ST : 0; l < gt; ++l) tc_drain(&k_full[l % ST], (l / ST) & 1);
      if (nu > 0) tc_drain(q_full, (nu - 1) & 1);
    }
  } else if (warp == 6) {
    // ------------------------------------------------------------------ V loader
    if (lane == 0) {
      uint32_t gt = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        const TcUnit w = tc_unit(u, chunks, chunk_len, N);
        for (int j = 0; j < w.tiles; ++j) {
          const uint32_t st = gt % ST;
          if (!(ok = tc_wait_nap(&v_empty[st], ((gt / ST) & 1) ^ 1, abort_flag, kNapLoad))) break;
          mbar_arrive_expect_tx(&v_full[st], C::kTile);
          for (int bx = 0; bx < C::kBoxes; ++bx)
            tma_load_3d(smem + C::kOffV + st * C::kTile + bx * C::kBox, &mv, &v_full[st], 64 * bx,
                        w.key_begin + j * kTileKeys, w.bh);
          ++gt;
        }
      }
      if (!ok)  // copies in flight land before the CTA can exit
        for (uint32_t l = gt > ST ? gt - ST : 0; l < gt; ++l) tc_drain(&v_full[l % ST], (l / ST) & 1);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint64_t dq = sdesc_sw128(smem_u32(smem + C::kOffQ), 16, 1024);
      const uint64_t dk = sdesc_sw128(smem_u32(smem + C::kOffK), 16, 1024);
      const uint64_t dv = sdesc_sw128(smem_u32(smem + C::kOffV), C::kBox, 1024);
      uint32_t gt = 0, nu = 0;
      bool ok = true;
      auto issue_pv = [&](uint32_t g, bool first) -> bool {
        const uint32_t b = g & 1, st = g % ST;
        if (!tc_wait_nap(&p_ready[b], (g >> 1) & 1, abort_flag, kNapIssue)) return false;
        if (!tc_wait_nap(&v_full[st], (g / ST) & 1, abort_flag, kNapIssue)) return false;
        tc_fence_after();
        mma_ts_k128(tmem + C::kColO, tmem + C::kColS + 128 * b, dv + ((st * C::kTile) >> 4),
                    C::kIdescPV, first ? 0u : 1u);
        tc_commit(o_done);
        tc_commit(&v_empty[st]);
        return true;
      };
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        const TcUnit w = tc_unit(u, chunks, chunk_len, N);
        if (w.tiles == 0) continue;
        if (!(ok = tc_wait_nap(q_full, nu & 1, abort_flag, kNapIssue))) break;
        fence_proxy_async_smem();  // Q came through cp.async (generic proxy)
        tc_fence_after();
        for (int j = 0; j < w.tiles; ++j, ++gt) {
          const uint32_t st = gt % ST, b = gt & 1;
          if (!(ok = tc_wait_nap(&k_full[st], (gt / ST) & 1, abort_flag, kNapIssue))) break;
          tc_fence_after();
          const uint64_t k0 = dk + ((st * C::kTile) >> 4);
          if constexpr (D == 64)
            mma_ss_k64(tmem + C::kColS + 128 * b, dq, k0, C::kIdescQK);
          else
            mma_ss_k128(tmem + C::kColS + 128 * b, dq, k0, C::kIdescQK, C::kBox >> 4);
          tc_commit(&s_full[b]);
          tc_commit(&k_empty[st]);
          if (j == w.tiles - 1) tc_commit(q_empty);  // the unit's last Q K^T
          if (j > 0 && !(ok = issue_pv(gt - 1, j == 1))) break;
        }
        if (!ok) break;
        if (!(ok = issue_pv(gt - 1, w.tiles == 1))) break;
        ++nu;
      }
      tc_commit(drain);  // every MMA completes before TMEM is released
      tc_drain(drain, 0);
    }
  } else {
    // ------------------------------------------------------------------ softmax
    const int variant = warp >> 1;          // 0 dense, 1 spatial
    const int r = (warp & 1) * 32 + lane;   // sampled row
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t t_o = tmem + lane_off + C::kColO;
    const int f = r < S ? clamp_index(idx[r], N) / P : 0;
    uint32_t gt = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
      const TcUnit w = tc_unit(u, chunks, chunk_len, N);
      if (w.tiles == 0) continue;
      // this row's keys in the range: [lo, hi), all of them (dense) or its
      // band of frames (spatial); empty for padding rows
      int lo = w.key_begin, hi = w.key_begin;
      if (r < S) {
        if (variant == 0) {
          hi = w.key_end;
        } else {
          lo = max(w.key_begin, max(0, f - width) * P);
          hi = static_cast<int>(min(static_cast<long long>(w.key_end),
                                    static_cast<long long>(f + width + 1) * P));
        }
      }
      // the warp's keys: tiles outside [wlo, whi) need no scores
      const int wlo = __reduce_min_sync(0xffffffffu, lo < hi ? lo : INT_MAX);
      const int whi = __reduce_max_sync(0xffffffffu, lo < hi ? hi : INT_MIN);
      float m = -INFINITY, lx = 0.f, ly = 0.f;
      for (int j = 0; j < w.tiles; ++j, ++gt) {
        const uint32_t b = gt & 1;
        const uint32_t t_s = tmem + lane_off + C::kColS + 128 * b;
        if (!(ok = tc_wait_warp(&s_full[b], (gt >> 1) & 1, abort_flag))) break;
        tc_fence_after();
        const int c0 = w.key_begin + j * kTileKeys;
        uint32_t p[4][16];
        if (c0 < whi && c0 + kTileKeys > wlo) {  // warp-uniform
          float s[128];
          {
            uint32_t rr[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld32(t_s + 32 * c, rr[c]);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              reg_fence32(rr[c]);
#pragma unroll
              for (int i = 0; i < 32; ++i) s[32 * c + i] = __uint_as_float(rr[c][i]);
            }
          }
          // the raw scores s; the scale (> 0) enters the max afterwards and
          // the exponent through one fused multiply-add.  This row's keys in
          // the tile are the columns [a0, a1): a row with none takes no part
          // (max -inf, weights 0); a warp-uniform -inf pass over the other
          // columns runs only where some row is cut inside the tile
          const int a0 = max(0, lo - c0), a1 = max(a0, min(kTileKeys, hi - c0));
          const bool none = a1 <= a0;
          if (__any_sync(0xffffffffu, !none && (a0 != 0 || a1 != kTileKeys))) {
#pragma unroll
            for (int i = 0; i < kTileKeys; ++i) s[i] = (i >= a0 && i < a1) ? s[i] : -INFINITY;
          }
          float m4[4] = {s[0], s[1], s[2], s[3]};
#pragma unroll
          for (int i = 4; i < 124; i += 8)
#pragma unroll
            for (int c = 0; c < 4; ++c) m4[c] = sm100::max3(m4[c], s[i + c], s[i + 4 + c]);
          const float mx = none ? -INFINITY
                                : sm100::max3(sm100::max3(m4[0], s[124], s[125]),
                                              sm100::max3(m4[1], s[126], s[127]),
                                              fmaxf(m4[2], m4[3])) * scale_log2;
          // lazy rescaling: the running max moves only when it grows by more
          // than 2^8
          float alpha = 1.f;
          bool need = false;
          if (mx > m + 8.f) {
            if (m != -INFINITY) {
              alpha = exp2f(m - mx);
              need = true;
            }
            m = mx;
          }
          lx *= alpha;
          ly *= alpha;
          // O may be rescaled once the previous tile's P.V finished (these
          // scores imply the P.V two tiles back did, so the barrier is at
          // most one phase ahead of this wait)
          if (__any_sync(0xffffffffu, need)) {
            if (!(ok = tc_wait_warp(o_done, (gt - 1) & 1, abort_flag))) break;
            tc_fence_after();
            uint32_t rr[32];
#pragma unroll
            for (int ch = 0; ch < D / 32; ++ch) {
              tmem_ld32(t_o + 32 * ch, rr);
              tmem_wait_ld();
              reg_fence32(rr);
#pragma unroll
              for (int i = 0; i < 32; ++i) rr[i] = __float_as_uint(__uint_as_float(rr[i]) * alpha);
              tmem_st32(t_o + 32 * ch, rr);
            }
          }
          // weights as bf16 pairs, exp2(s * scale - m); a row with no key in
          // the tile, or none yet, takes -inf as the offset (weights 0); the
          // row sums add the rounded weights the tensor core sees
          const float neg = (none || m == -INFINITY) ? -INFINITY : -m;
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const int k = 32 * c + 2 * i;
              float t0, t1;
              sm100::fma2(t0, t1, s[k], s[k + 1], scale_log2, scale_log2, neg, neg);
              p[c][i] = pack_bf16x2(fast_exp2(t0), fast_exp2(t1));
              lx += __uint_as_float(p[c][i] << 16);
              ly += __uint_as_float(p[c][i] & 0xffff0000u);
            }
        } else {
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int i = 0; i < 16; ++i) p[c][i] = 0u;
        }
        // (tcgen05.st and wait::st are warp-wide: the lanes meet first)
        __syncwarp();
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_st16(t_s + 16 * c, p[c]);
        tmem_wait_st();
        // before the unit's last weights are released, the P.V before them
        // has finished: o_done then stands at most one phase past what the
        // epilogue waits for (two would alias its parity)
        if (j == w.tiles - 1 && gt > 0 && !(ok = tc_wait_warp(o_done, (gt - 1) & 1, abort_flag)))
          break;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_ready[b]);
      }
      if (!ok) break;
      // the unit's state rows; o_done completes one phase per tile's P.V and
      // the one before the last has finished, so a single wait finds the last
      if (!(ok = tc_wait_warp(o_done, (gt - 1) & 1, abort_flag))) break;
      tc_fence_after();
      float* row = tc_state_row<D>(ws, w, variant, r, chunks);
      row[0] = m;
      row[1] = lx + ly;
      uint32_t rr[32];
#pragma unroll
      for (int ch = 0; ch < D / 32; ++ch) {
        tmem_ld32(t_o + 32 * ch, rr);
        tmem_wait_ld();
        reg_fence32(rr);
#pragma unroll
        for (int i = 0; i < 32; ++i) row[2 + 32 * ch + i] = __uint_as_float(rr[i]);
      }
      // (the next unit's first P.V overwrites O only after this warp's next
      // p_ready, which follows these reads in program order)
    }
    if (!ok) {
      // a wait gave up: this CTA's results are not to be trusted
      for (int u = blockIdx.x; u < n_units; u += gridDim.x)
        tc_state_row<D>(ws, tc_unit(u, chunks, chunk_len, N), variant, r, chunks)[0] =
            __int_as_float(0x7fc00000);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 5) tmem_dealloc(tmem, 512);
}

// --------------------------------------------------------------- combine

template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) {
  return x;
}
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}

constexpr int kMergeRows = 4;      // sampled rows per merge CTA (one warp each)
constexpr int kTemporalBatch = 8;  // temporal keys whose loads are in flight together

// Merges the chunk states of one sampled row (one warp per row), computes the
// row's temporal output directly and writes the row's squared errors.
template <int D, typename T>
__global__ void __launch_bounds__(32 * kMergeRows) profile_merge(
    const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
    const int32_t* __restrict__ idx, int S, int N, int F, int P, float scale_log2, int chunks,
    const float* __restrict__ ws, float* __restrict__ errs) {
  constexpr int E = D / 32;
  const int bh = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.y * kMergeRows + warp;
  if (r >= kRows) return;
  float* err = errs + (static_cast<long long>(bh) * kRows + r) * 2;
  if (r >= S) {
    if (lane == 0) err[0] = err[1] = 0.f;
    return;
  }
  const long long head = static_cast<long long>(bh) * N * D;
  const int stride = kRows * state_floats<D>();  // between chunks
  float om[2][E];
#pragma unroll
  for (int var = 0; var < 2; ++var) {
    const float* st = ws + (static_cast<long long>(bh) * 2 + var) * chunks * stride +
                      static_cast<long long>(r) * state_floats<D>();
    // lane c holds chunk c's weight exp2(m_c - M) / sum_c exp2(m_c - M) l_c
    const float mc = lane < chunks ? st[static_cast<long long>(lane) * stride] : -INFINITY;
    float M = mc;
#pragma unroll
    for (int o2 = 16; o2 > 0; o2 >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o2));
    float w = mc == -INFINITY ? 0.f : exp2f(mc - M);
    float L = lane < chunks ? w * st[static_cast<long long>(lane) * stride + 1] : 0.f;
#pragma unroll
    for (int o2 = 16; o2 > 0; o2 >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o2);
    w = L > 0.f ? w / L : 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) om[var][e] = 0.f;
    for (int c = 0; c < chunks; ++c) {
      const float wc = __shfl_sync(0xffffffffu, w, c);
      const float* oc = st + static_cast<long long>(c) * stride + 2;
#pragma unroll
      for (int e = 0; e < E; ++e) om[var][e] = fmaf(wc, oc[lane + 32 * e], om[var][e]);
    }
  }
  // temporal mask: the F keys of the row's position, exact online softmax
  const int n = clamp_index(idx[r], N);
  const int sp = n % P;
  float qv[E], acc[E], m = -INFINITY, l = 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    qv[e] = to_f(q[head + static_cast<long long>(n) * D + lane + 32 * e]);
    acc[e] = 0.f;
  }
  // keys in groups of kTemporalBatch: all their K and V loads are issued
  // before any of them is used, so the group costs one memory latency
  for (int f0 = 0; f0 < F; f0 += kTemporalBatch) {
    float kx[kTemporalBatch][E], vx[kTemporalBatch][E];
#pragma unroll
    for (int b = 0; b < kTemporalBatch; ++b) {
      const int f = min(f0 + b, F - 1);
      const long long j = static_cast<long long>(f) * P + sp;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        kx[b][e] = to_f(k[head + j * D + lane + 32 * e]);
        vx[b][e] = to_f(v[head + j * D + lane + 32 * e]);
      }
    }
#pragma unroll
    for (int b = 0; b < kTemporalBatch; ++b) {
      if (f0 + b >= F) break;
      float dot = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) dot = fmaf(qv[e], kx[b][e], dot);
#pragma unroll
      for (int o2 = 16; o2 > 0; o2 >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o2);
      const float t = dot * scale_log2;
      const float mn = fmaxf(m, t);
      const float alpha = exp2f(m - mn);
      const float p = exp2f(t - mn);
      l = l * alpha + p;
#pragma unroll
      for (int e = 0; e < E; ++e) acc[e] = fmaf(p, vx[b][e], acc[e] * alpha);
      m = mn;
    }
  }
  float es = 0.f, et = 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const float ds = om[1][e] - om[0][e], dt = acc[e] / l - om[0][e];
    es = fmaf(ds, ds, es);
    et = fmaf(dt, dt, et);
  }
#pragma unroll
  for (int o2 = 16; o2 > 0; o2 >>= 1) {
    es += __shfl_xor_sync(0xffffffffu, es, o2);
    et += __shfl_xor_sync(0xffffffffu, et, o2);
  }
  if (lane == 0) {
    err[0] = es;
    err[1] = et;
  }
}

// Per head: mean squared errors over the S x d sampled outputs and the mode.
__global__ void __launch_bounds__(kRows) profile_finalize(const float* __restrict__ errs, int S,
                                                          int D, float* __restrict__ mse_out,
                                                          int32_t* __restrict__ mode_out) {
  __shared__ float red[2][2];
  const int bh = blockIdx.x, r = threadIdx.x, lane = r & 31, warp = r >> 5;
  float es = 0.f, et = 0.f;
  if (r < S) {
    es = errs[(static_cast<long long>(bh) * kRows + r) * 2];
    et = errs[(static_cast<long long>(bh) * kRows + r) * 2 + 1];
  }
#pragma unroll
  for (int o2 = 16; o2 > 0; o2 >>= 1) {
    es += __shfl_xor_sync(0xffffffffu, es, o2);
    et += __shfl_xor_sync(0xffffffffu, et, o2);
  }
  if (lane == 0) {
    red[0][warp] = es;
    red[1][warp] = et;
  }
  __syncthreads();
  if (r == 0) {
    const float denom = static_cast<float>(S) * D;
    es = (red[0][0] + red[0][1]) / denom;
    et = (red[1][0] + red[1][1]) / denom;
    if (mse_out != nullptr) {
      mse_out[2 * bh] = es;
      mse_out[2 * bh + 1] = et;
    }
    mode_out[bh] = et < es ? SVG_MODE_TEMPORAL : SVG_MODE_SPATIAL;
  }
}

// Launches partial + combine with the given key chunking and state buffer.
template <int D>
svg_status launch_profile_shaped(const void* q, const void* k, const void* v, int dtype, int B,
                                 int H, int N, int F, int P, int width, const int32_t* idx, int S,
                                 float* mse_out, int32_t* mode_out, float* ws, ProfileShape ps,
                                 cudaStream_t s, const char* who) {
  const float scale_log2 = kLog2e / sqrtf(static_cast<float>(D));
  float* errs = ws + states_bytes(B, H, ps.chunks, D) / sizeof(float);
  if (dtype == SVG_BF16) {
    using C = TcCfg<D>;
    CUtensorMap mk, mv;
    if (!make_tma_map_3d(&mk, k, B * H, N, D) || !make_tma_map_3d(&mv, v, B * H, N, D))
      return fail(SVG_ERR_CUDA, "%s: cannot encode TMA descriptors", who);
    if (cudaFuncSetAttribute(profile_partial_tc<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::kSmem) != cudaSuccess)
      return fail(SVG_ERR_CUDA, "%s: cannot reserve shared memory", who);
    const int units = ps.chunks * B * H;
    const int grid = units < sm_count() ? units : sm_count();
    profile_partial_tc<D><<<grid, kTcThreads, C::kSmem, s>>>(
        mk, mv, static_cast<const __nv_bfloat16*>(q), idx, S, N, P, width, scale_log2, ps.chunks,
        ps.chunk_len, units, ws);
    if (svg_status st = check_launch(who)) return st;
    profile_merge<D, __nv_bfloat16><<<dim3(B * H, kRows / kMergeRows), 32 * kMergeRows, 0, s>>>(
        static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
        static_cast<const __nv_bfloat16*>(v), idx, S, N, F, P, scale_log2, ps.chunks, ws, errs);
  } else {
    profile_partial_fp32<D><<<dim3(ps.chunks, B * H, 2), 256, 0, s>>>(
        static_cast<const float*>(q), static_cast<const float*>(k), static_cast<const float*>(v),
        idx, S, N, P, width, scale_log2, ps.chunks, ps.chunk_len, ws);
    if (svg_status st = check_launch(who)) return st;
    profile_merge<D, float><<<dim3(B * H, kRows / kMergeRows), 32 * kMergeRows, 0, s>>>(
        static_cast<const float*>(q), static_cast<const float*>(k), static_cast<const float*>(v),
        idx, S, N, F, P, scale_log2, ps.chunks, ws, errs);
  }
  if (svg_status st = check_launch(who)) return st;
  profile_finalize<<<B * H, kRows, 0, s>>>(errs, S, D, mse_out, mode_out);
  return check_launch(who);
}

}  // namespace
}  // namespace svg

using namespace svg;

extern "C" size_t svg_profile_workspace_size(int B, int H, int N, int d, int S) {
  if (B <= 0 || H <= 0 || N <= 0 || (d != 64 && d != 128) || S <= 0) return 0;
  return (partial_bytes(B, H, N, d) + 255) / 256 * 256;
}

extern "C" svg_status svg_profile_heads(const void* q, const void* k, const void* v, int dtype,
                                        int B, int H, int N, int d, int frames,
                                        int tokens_per_frame, int spatial_width,
                                        const int32_t* sample_idx, int S, float* mse_out,
                                        int32_t* mode_out, void* workspace, size_t workspace_bytes,
                                        void* stream) {
  clear_error();
  if (q == nullptr || k == nullptr || v == nullptr || sample_idx == nullptr || mode_out == nullptr)
    return fail(SVG_ERR_INVALID_ARG, "profile: null pointer");
  if (dtype != SVG_BF16 && dtype != SVG_FP32)
    return fail(SVG_ERR_INVALID_ARG, "profile: bad dtype %d", dtype);
  if (B <= 0 || H <= 0 || N <= 0 || B * H > 65535)
    return fail(SVG_ERR_INVALID_ARG, "profile: bad shape");
  if (d != 64 && d != 128) return fail(SVG_ERR_INVALID_ARG, "profile: d=%d not in {64,128}", d);
  if (frames <= 0 || tokens_per_frame <= 0 || static_cast<long long>(frames) * tokens_per_frame != N)
    return fail(SVG_ERR_INVALID_ARG, "profile: frames*tokens_per_frame != N");
  if (spatial_width < 0) return fail(SVG_ERR_INVALID_ARG, "profile: spatial_width < 0");
  if (S < 1 || S > kRows) return fail(SVG_ERR_INVALID_ARG, "profile: S=%d not in [1,%d]", S, kRows);
  if (!aligned16(q) || !aligned16(k) || !aligned16(v))
    return fail(SVG_ERR_INVALID_ARG, "profile: tensors must be 16-byte aligned");
  if (workspace == nullptr || !aligned256(workspace) ||
      workspace_bytes < svg_profile_workspace_size(B, H, N, d, S))
    return fail(SVG_ERR_INVALID_ARG, "profile: workspace too small or not 256-byte aligned");
  auto* ws = static_cast<float*>(workspace);
  cudaStream_t s = as_stream(stream);
  const ProfileShape ps = profile_shape(B, H, N);
  if (d == 64)
    return launch_profile_shaped<64>(q, k, v, dtype, B, H, N, frames, tokens_per_frame,
                                     spatial_width, sample_idx, S, mse_out, mode_out, ws, ps, s,
                                     "profile");
  return launch_profile_shaped<128>(q, k, v, dtype, B, H, N, frames, tokens_per_frame,
                                    spatial_width, sample_idx, S, mse_out, mode_out, ws, ps, s,
                                    "profile");
}

// ---------------------------------------------------------------------------
// Allocation-free variant: svg_profile_heads_noalloc.
//
// Some callers cannot allocate device memory at all: a plugin running inside
// an engine that owns every byte of device memory and hands out no
// workspace, or a latency-critical or captured region of a program where a
// cudaMalloc would synchronise the device or is not permitted.  For them the
// profiling scratch (the per-chunk online-softmax states) lives in one
// fixed-size array in device global memory that belongs to this library.
// Its size is a compile-time constant; every GPU that loads the library
// holds it until the process exits.
// ---------------------------------------------------------------------------

#include <mutex>

namespace svg {
namespace {

constexpr size_t kFixedScratchBytes = size_t(16) << 20;  // 16 MiB

// The library-owned scratch.  Host code must not pass this symbol itself to
// a kernel (on the host it is only a stand-in); it uses the device address
// that cudaGetSymbolAddress returns for the current device.
static __device__ __align__(256) unsigned char g_profile_scratch[kFixedScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {nullptr};

// Device address of g_profile_scratch on the current device, looked up once
// per device on first use.
svg_status fixed_scratch(float** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(SVG_ERR_CUDA, "profile_noalloc: cudaGetDevice: %s",
                                    cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices)
    return fail(SVG_ERR_UNSUPPORTED, "profile_noalloc: device index %d >= %d", dev, kMaxDevices);
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_profile_scratch);
    if (e != cudaSuccess || p == nullptr)
      return fail(SVG_ERR_CUDA, "profile_noalloc: cudaGetSymbolAddress: %s", cudaGetErrorString(e));
    g_scratch_addr[dev] = p;
  }
  *out = static_cast<float*>(g_scratch_addr[dev]);
  return SVG_OK;
}

// Bytes of scratch one key range (chunk) of every head needs.
size_t fixed_bytes_per_chunk(int B, int H, int d) {
  return static_cast<size_t>(B) * H * 2 * kRows * (d + 2) * sizeof(float);
}

// Scratch left for the chunk states after the per-row error sums.
size_t fixed_state_budget(int B, int H) {
  const size_t e = errors_bytes(B, H) + 256;  // + rounding of the state region
  return e < kFixedScratchBytes ? kFixedScratchBytes - e : 0;
}

// The chunking of profile_shape, reduced until the states fit the fixed
// scratch (fewer, longer key ranges per head).
ProfileShape fixed_shape(int B, int H, int N, int d) {
  ProfileShape ps = profile_shape(B, H, N);
  const long long max_chunks =
      static_cast<long long>(fixed_state_budget(B, H) / fixed_bytes_per_chunk(B, H, d));
  if (ps.chunks > max_chunks) ps = shape_for(N, max_chunks);
  return ps;
}

}  // namespace
}  // namespace svg

extern "C" svg_status svg_profile_heads_noalloc(const void* q, const void* k, const void* v,
                                                int dtype, int B, int H, int N, int d, int frames,
                                                int tokens_per_frame, int spatial_width,
                                                const int32_t* sample_idx, int S, float* mse_out,
                                                int32_t* mode_out, void* stream) {
  clear_error();
  if (q == nullptr || k == nullptr || v == nullptr || sample_idx == nullptr || mode_out == nullptr)
    return fail(SVG_ERR_INVALID_ARG, "profile_noalloc: null pointer");
  if (dtype != SVG_BF16 && dtype != SVG_FP32)
    return fail(SVG_ERR_INVALID_ARG, "profile_noalloc: bad dtype %d", dtype);
  if (B <= 0 || H <= 0 || N <= 0 || B * H > 65535)
    return fail(SVG_ERR_INVALID_ARG, "profile_noalloc: bad shape");
  if (d != 64 && d != 128)
    return fail(SVG_ERR_INVALID_ARG, "profile_noalloc: d=%d not in {64,128}", d);
  if (frames <= 0 || tokens_per_frame <= 0 || static_cast<long long>(frames) * tokens_per_frame != N)
    return fail(SVG_ERR_INVALID_ARG, "profile_noalloc: frames*tokens_per_frame != N");
  if (spatial_width < 0) return fail(SVG_ERR_INVALID_ARG, "profile_noalloc: spatial_width < 0");
  if (S < 1 || S > kRows)
    return fail(SVG_ERR_INVALID_ARG, "profile_noalloc: S=%d not in [1,%d]", S, kRows);
  if (!aligned16(q) || !aligned16(k) || !aligned16(v))
    return fail(SVG_ERR_INVALID_ARG, "profile_noalloc: tensors must be 16-byte aligned");
  if (fixed_bytes_per_chunk(B, H, d) > fixed_state_budget(B, H))
    return fail(SVG_ERR_INVALID_ARG,
                "profile_noalloc: B*H=%d heads at d=%d need %zu bytes of scratch per key range; the "
                "fixed scratch holds %zu bytes (at most %zu heads)",
                B * H, d, fixed_bytes_per_chunk(B, H, d) + errors_bytes(B, H), kFixedScratchBytes,
                kFixedScratchBytes / (fixed_bytes_per_chunk(1, 1, d) + kRows * 2 * sizeof(float)));
  float* ws = nullptr;
  if (svg_status st = fixed_scratch(&ws)) return st;
  cudaStream_t s = as_stream(stream);
  const ProfileShape ps = fixed_shape(B, H, N, d);
  if (d == 64)
    return launch_profile_shaped<64>(q, k, v, dtype, B, H, N, frames, tokens_per_frame,
                                     spatial_width, sample_idx, S, mse_out, mode_out, ws, ps, s,
                                     "profile_noalloc");
  return launch_profile_shaped<128>(q, k, v, dtype, B, H, N, frames, tokens_per_frame,
                                    spatial_width, sample_idx, S, mse_out, mode_out, ws, ps, s,
                                    "profile_noalloc");
}
