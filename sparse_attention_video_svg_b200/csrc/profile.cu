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
//   partial  grid (chunks, B*H): the keys of a head are cut into `chunks`
//            contiguous ranges.  A CTA of 4 warps streams one range through
//            a cp.async ring (4 stages of 64 keys at d = 64, 3 at d = 128);
//            each warp owns 16 of the 64 sampled rows and keeps two
//            online-softmax states (max, sum, o) for them: dense and under
//            the spatial mask (each row's band of frames is one contiguous
//            key range, tested with two compares; the spatial update is
//            skipped for stages outside the warp's bands).  Both updates
//            share one Q K^T per stage.  bf16: mma.sync tensor-core products;
//            fp32: SIMT (one launch per mask, grid z).
//   merge    grid (B*H, 16), one warp per sampled row: the chunk weights
//            exp2(m_c - M) / L, the merged dense and spatial outputs, the
//            temporal output (a row sees only the F keys of its position,
//            computed directly) and the row's squared errors;
//   finalize grid (B*H): mean errors and the mode.
// The pass reads K and V once per head and costs a few percent of the
// attention it configures.
#include <float.h>

#include "common.cuh"
#include "mma_frag.cuh"

namespace svg {
namespace {

constexpr int kRows = 64;          // sampled rows per head (S padded to 64)
constexpr int kKeys = 64;          // keys per shared-memory stage
constexpr int kThreads = 128;      // bf16 partial: 4 warps, 16 rows each
constexpr int kTargetCtas = 888;   // partial-grid size the chunking aims for (6 x 148)
constexpr int kMaxChunks = 32;     // merge holds one chunk weight per lane
constexpr float kLog2e = 1.4426950408889634f;

// Sampled indices outside [0, N) are clamped into range (never read out of bounds).
__device__ __forceinline__ int clamp_index(int n, int N) { return n < 0 ? 0 : (n >= N ? N - 1 : n); }

struct ProfileShape {
  int chunks;     // key ranges per head
  int chunk_len;  // keys per range (multiple of kKeys)
};

ProfileShape shape_for(int N, long long chunks) {
  const long long max_chunks = (N + 4 * kKeys - 1) / (4 * kKeys);  // >= 4 stages per range
  if (chunks > max_chunks) chunks = max_chunks;
  if (chunks > kMaxChunks) chunks = kMaxChunks;
  if (chunks < 1) chunks = 1;
  long long len = (N + chunks - 1) / chunks;
  len = (len + kKeys - 1) / kKeys * kKeys;
  chunks = (N + len - 1) / len;
  return {static_cast<int>(chunks), static_cast<int>(len)};
}

ProfileShape profile_shape(int B, int H, int N) {
  const long long bh = static_cast<long long>(B) * H;
  return shape_for(N, (kTargetCtas + bh - 1) / bh);
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

// --------------------------------------------------------------- bf16 partial

template <int D>
constexpr int stages_for() {
  return D == 64 ? 4 : 3;  // cp.async ring depth (shared memory: 3 or 2 CTAs per SM)
}
template <int D>
constexpr size_t partial_smem() {
  return static_cast<size_t>(kRows) * D * 2 + 2 * static_cast<size_t>(stages_for<D>()) * kKeys * D * 2;
}

// One stage's online-softmax update of a warp's 16 rows: s holds the scores
// (scale * log2 e applied below), keys outside [lo[h], hi[h]) are masked for
// the thread's row h; P is rounded to bf16 and the row sum adds the rounded
// values.
template <int D>
__device__ __forceinline__ void stage_update(float (&m)[2], float (&l)[2], float (&o)[D / 8][4],
                                             float (&s)[kKeys / 8][4], const int (&lo)[2],
                                             const int (&hi)[2], int key0, float scale_log2,
                                             uint32_t vtile) {
  const int t4 = threadIdx.x & 3;
  float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
  for (int n = 0; n < kKeys / 8; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int key = key0 + 8 * n + 2 * t4 + (e & 1);
      const int h = e >> 1;
      s[n][e] = (key >= lo[h] && key < hi[h]) ? s[n][e] * scale_log2 : -INFINITY;
      mx[h] = fmaxf(mx[h], s[n][e]);
    }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
    mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
    const float mn = fmaxf(m[h], mx[h]);
    const float base = mn == -INFINITY ? 0.f : mn;
    const float alpha = fast_exp2(m[h] - base);  // exp2(-inf) = 0 on the first update
    m[h] = mn;
    l[h] *= alpha;
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
      o[n][2 * h] *= alpha;
      o[n][2 * h + 1] *= alpha;
    }
#pragma unroll
    for (int n = 0; n < kKeys / 8; ++n) {
      s[n][2 * h] = round_bf16(fast_exp2(s[n][2 * h] - base));
      s[n][2 * h + 1] = round_bf16(fast_exp2(s[n][2 * h + 1] - base));
      l[h] += s[n][2 * h] + s[n][2 * h + 1];
    }
  }
  pv_frags<D, kKeys>(o, s, vtile, 0);
}

template <int D>
__device__ __forceinline__ void store_state(float* base, int row0, const float (&m)[2],
                                            float (&l)[2], const float (&o)[D / 8][4]) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t4 = lane & 3;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    l[h] += __shfl_xor_sync(0xffffffffu, l[h], 1);
    l[h] += __shfl_xor_sync(0xffffffffu, l[h], 2);
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float* row = base + (row0 + g + 8 * h) * state_floats<D>();
    if (t4 == 0) {
      row[0] = m[h];
      row[1] = l[h];
    }
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
      row[2 + 8 * n + 2 * t4] = o[n][2 * h];
      row[2 + 8 * n + 2 * t4 + 1] = o[n][2 * h + 1];
    }
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads, D == 64 ? 3 : 2) profile_partial_bf16(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
    const __nv_bfloat16* __restrict__ v, const int32_t* __restrict__ idx, int S, int N, int P,
    int width, float scale_log2, int chunks, int chunk_len, float* __restrict__ ws) {
  constexpr int ST = stages_for<D>();
  constexpr int TILE = kKeys * D * 2;  // bytes of one K or V stage
  extern __shared__ __align__(128) unsigned char smem[];
  unsigned char* sQ = smem;
  unsigned char* sK = smem + kRows * D * 2;
  unsigned char* sV = sK + ST * TILE;

  const int chunk = blockIdx.x, bh = blockIdx.y;
  const long long head = static_cast<long long>(bh) * N * D;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row0 = warp * 16;
  const int g = lane >> 2;
  const int key_begin = chunk * chunk_len;
  const int key_end = min(N, key_begin + chunk_len);
  const int n_stages = (key_end - key_begin + kKeys - 1) / kKeys;

  // gather the sampled query rows (padding rows are zero)
  for (int t = threadIdx.x; t < kRows * (D / 8); t += kThreads) {
    const int r = t / (D / 8), c = t % (D / 8);
    const bool ok = r < S;
    const int n = ok ? clamp_index(idx[r], N) : 0;
    cp_async16(sQ + swz(r, c, 2 * D), q + head + static_cast<long long>(n) * D + c * 8, ok);
  }
  // the keys each of this thread's two rows may see, clipped to the chunk:
  // every key of the chunk (dense) and the row's band of frames (spatial)
  int dlo[2], dhi[2], slo[2], shi[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int r = row0 + g + 8 * h;
    dlo[h] = slo[h] = key_begin;
    dhi[h] = shi[h] = key_end;
    if (r >= S) {
      dhi[h] = shi[h] = key_begin;  // padding row: no keys
    } else {
      const int f = clamp_index(idx[r], N) / P;
      slo[h] = max(key_begin, max(0, f - width) * P);
      shi[h] = min(key_end, static_cast<int>(min(static_cast<long long>(N),
                                                 static_cast<long long>(f + width + 1) * P)));
    }
  }
  int wlo = min(slo[0], slo[1]), whi = max(shi[0], shi[1]);
#pragma unroll
  for (int o2 = 4; o2 < 32; o2 <<= 1) {
    wlo = min(wlo, __shfl_xor_sync(0xffffffffu, wlo, o2));
    whi = max(whi, __shfl_xor_sync(0xffffffffu, whi, o2));
  }

#pragma unroll
  for (int st = 0; st < ST - 1; ++st) {
    if (st < n_stages) {
      load_tile_async<D, kKeys, kThreads>(sK + st * TILE, k + head, key_begin + st * kKeys, key_end);
      load_tile_async<D, kKeys, kThreads>(sV + st * TILE, v + head, key_begin + st * kKeys, key_end);
    }
    cp_async_commit();
  }

  float md[2] = {-INFINITY, -INFINITY}, ld[2] = {0.f, 0.f};
  float ms[2] = {-INFINITY, -INFINITY}, ls[2] = {0.f, 0.f};
  float od[D / 8][4], os[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) od[n][e] = os[n][e] = 0.f;
  uint32_t qa[D / 16][4];

  for (int st = 0; st < n_stages; ++st) {
    cp_async_wait<ST - 2>();
    __syncthreads();  // stage st landed; the buffer refilled below is free
    {
      const int ns = st + ST - 1;
      if (ns < n_stages) {
        const int b = ns % ST;
        load_tile_async<D, kKeys, kThreads>(sK + b * TILE, k + head, key_begin + ns * kKeys, key_end);
        load_tile_async<D, kKeys, kThreads>(sV + b * TILE, v + head, key_begin + ns * kKeys, key_end);
      }
      cp_async_commit();
    }
    if (st == 0) load_a_frags<D>(qa, smem_u32(sQ), row0);
    const int key0 = key_begin + st * kKeys;
    const int b = st % ST;
    float s[kKeys / 8][4];
    qk_frags<D, kKeys>(s, qa, smem_u32(sK + b * TILE), 0);
    if (key0 < whi && key0 + kKeys > wlo) {  // some row of this warp has band keys here
      float sp[kKeys / 8][4];
#pragma unroll
      for (int n = 0; n < kKeys / 8; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) sp[n][e] = s[n][e];
      stage_update<D>(ms, ls, os, sp, slo, shi, key0, scale_log2, smem_u32(sV + b * TILE));
    }
    stage_update<D>(md, ld, od, s, dlo, dhi, key0, scale_log2, smem_u32(sV + b * TILE));
  }

  // per-row partial states -> workspace [bh][variant][chunk][row][m, l, o[D]]
  const long long stride = static_cast<long long>(chunks) * kRows * state_floats<D>();
  float* base = ws + (static_cast<long long>(bh) * 2 * chunks + chunk) * kRows * state_floats<D>();
  store_state<D>(base, row0, md, ld, od);
  store_state<D>(base + stride, row0, ms, ls, os);
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
    const size_t smem = partial_smem<D>();
    if (cudaFuncSetAttribute(profile_partial_bf16<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return fail(SVG_ERR_CUDA, "%s: cannot reserve shared memory", who);
    profile_partial_bf16<D><<<dim3(ps.chunks, B * H), kThreads, smem, s>>>(
        static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
        static_cast<const __nv_bfloat16*>(v), idx, S, N, P, width, scale_log2, ps.chunks,
        ps.chunk_len, ws);
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
