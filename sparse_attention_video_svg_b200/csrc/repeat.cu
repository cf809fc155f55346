// Spatial-repetition heads.
//
// CalibAtt article (lpnh.cn/news/568491), section 3.2: in some heads the
// image rows of a frame attend almost identically.  Such a head is found by
// the mean cosine similarity of its rows' attention patterns (above
// gamma = 0.87); for it only k = 5 equally spaced anchor rows per frame are
// computed and every other row takes its anchor's output.
//
//   svg_row_similarity  per head: mean over the evaluated frames of the mean
//                       pairwise cosine between rows.  The pattern of row y
//                       of frame f is the pw x N block of dense attention
//                       probabilities of its tokens f P + y pw + x.
//                       Pass 1: log-sum-exp of the frames' query rows.
//                       Pass 2: per (head, frame, group of columns) the Gram
//                       matrix G[y][y'] = sum_x sum_j p(y,x),j p(y',x),j,
//                       scores on bf16 mma.sync, probabilities stored as
//                       fp16 and multiplied on fp16 mma.sync.
//                       Pass 3: cosines and means (fixed order).
//   svg_anchor_lists    the given lists followed by copies in which query
//                       tiles without an anchor-row token are empty, list
//                       ids moved to the copies for repeating heads, and a
//                       pairing order that puts the tiles with work first
//                       (anchor rows can fall in every other query tile,
//                       which would leave one tile of each work pair idle).
//   svg_row_broadcast   in place: each non-anchor row of a repeating head
//                       takes its anchor row's output.
//
// Anchors: the ph rows fall into k bands (band j = rows y with
// floor(y k / ph) = j); the anchor of a band is its middle row (the upper of
// two).
#include "common.cuh"
#include "mma_frag.cuh"

namespace svg {
namespace {

constexpr int kThreads = 256;
constexpr int kRows = 128;      // query rows per CTA
constexpr int kKeys = 64;       // keys per stage
constexpr int kMaxBlocks = 16;  // 16 x 8 Gram blocks per warp
constexpr float kLog2e = 1.4426950408889634f;

// ------------------------------------------------------------------ anchors

__host__ __device__ inline int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Anchor row of row y (y itself when every row is an anchor).
__host__ __device__ inline int anchor_of(int y, int ph, int k) {
  if (k >= ph) return y;
  const int j = y * k / ph;
  const int lo = ceil_div(j * ph, k), hi = ceil_div((j + 1) * ph, k);
  return lo + (hi - lo) / 2;
}

// ------------------------------------------------------- row similarity: lse

__device__ __forceinline__ int eval_frame(const int32_t* frames, int fi, int F, int32_t* status) {
  int f = frames != nullptr ? frames[fi] : fi;
  if (f < 0 || f >= F) {
    if (threadIdx.x == 0) set_status(status, SVG_DEVICE_BAD_INDEX);
    f = f < 0 ? 0 : F - 1;
  }
  return f;
}

struct RsArgs {
  const void* q;
  const void* k;
  const int32_t* frames;  // [nf] or null (frames 0 .. nf-1)
  float* lse;             // [BH][nf][P]
  float* gram;            // [BH][nf][ng][ph (ph + 1) / 2]
  float* sim;             // [BH]
  int32_t* status;
  int N, F, ph, pw, P, nf, ng, gx;  // gx columns per Gram CTA
  float scale_log2;
};

// Log2-sum-exp of the scaled scores of the frames' query rows over all N
// keys: a CTA takes 128 consecutive tokens of one evaluated frame.
template <int D>
__global__ void __launch_bounds__(kThreads) rs_lse_bf16(const RsArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  constexpr int TILE = kKeys * D * 2;
  unsigned char* sQ = smem;
  unsigned char* sK = smem + kRows * D * 2;
  const int r0 = blockIdx.x * kRows, fi = blockIdx.y, bh = blockIdx.z;
  const int f = eval_frame(a.frames, fi, a.F, a.status);
  const int N = a.N;
  const auto* q = static_cast<const __nv_bfloat16*>(a.q) + (static_cast<long long>(bh) * N +
                                                            static_cast<long long>(f) * a.P) * D;
  const auto* k = static_cast<const __nv_bfloat16*>(a.k) + static_cast<long long>(bh) * N * D;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t4 = lane & 3;
  load_tile_async<D, kRows, kThreads>(sQ, q, r0, a.P);
  load_tile_async<D, kKeys, kThreads>(sK, k, 0, N);
  cp_async_commit();
  float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};
  uint32_t qa[D / 16][4];
  const int n_stages = ceil_div(N, kKeys);
  for (int st = 0; st < n_stages; ++st) {
    if (st + 1 < n_stages) {
      load_tile_async<D, kKeys, kThreads>(sK + ((st + 1) & 1) * TILE, k, (st + 1) * kKeys, N);
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
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int n = 0; n < kKeys / 8; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const bool ok = key0 + 8 * n + 2 * t4 + (e & 1) < N;
        s[n][e] = ok ? s[n][e] * a.scale_log2 : -INFINITY;
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
    __syncthreads();
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    lrow[h] += __shfl_xor_sync(0xffffffffu, lrow[h], 1);
    lrow[h] += __shfl_xor_sync(0xffffffffu, lrow[h], 2);
    const int r = r0 + warp * 16 + g + 8 * h;
    if (t4 == 0 && r < a.P)
      a.lse[(static_cast<long long>(bh) * a.nf + fi) * a.P + r] = mrow[h] + __log2f(lrow[h]);
  }
}

// --------------------------------------------------- row similarity: Gram

__device__ __forceinline__ void mma_f16_16816(float* d, const uint32_t* a, const uint32_t* b) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

__device__ __forceinline__ void ldmatrix_x2(uint32_t& r0, uint32_t& r1, uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];\n"
               : "=r"(r0), "=r"(r1)
               : "r"(addr));
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ int tri_index(int y, int y2, int ph) {  // y <= y2
  return y * ph - y * (y - 1) / 2 + (y2 - y);
}

// Gram matrix of the rows of one group of columns of one evaluated frame.
// Tile row r = xl * ph + y holds token f P + y pw + (x0 + xl).
template <int D>
__global__ void __launch_bounds__(kThreads) rs_gram_bf16(const RsArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  constexpr int TILE = kKeys * D * 2;
  constexpr int PROW = kKeys * 2;  // bytes per probability row (64 fp16)
  unsigned char* sQ = smem;
  unsigned char* sK = sQ + kRows * D * 2;
  unsigned char* sP = sK + 2 * TILE;                       // [128][64] fp16, swizzled
  unsigned char* sZ = sP + kRows * PROW;                   // one zero row
  float* sL = reinterpret_cast<float*>(sZ + PROW);         // [128] lse
  float* sG = sL + kRows;                                  // [ph (ph + 1) / 2]
  const int grp = blockIdx.x, fi = blockIdx.y, bh = blockIdx.z;
  const int f = eval_frame(a.frames, fi, a.F, a.status);
  const int N = a.N, ph = a.ph, pw = a.pw, P = a.P;
  const int x0 = grp * a.gx, nx = min(a.gx, pw - x0), rows = nx * ph;
  const int tri = ph * (ph + 1) / 2;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t4 = lane & 3;
  const auto* qh = static_cast<const __nv_bfloat16*>(a.q) + static_cast<long long>(bh) * N * D;
  const auto* k = static_cast<const __nv_bfloat16*>(a.k) + static_cast<long long>(bh) * N * D;
  const float* lse = a.lse + (static_cast<long long>(bh) * a.nf + fi) * P;

  for (int i = threadIdx.x; i < tri; i += kThreads) sG[i] = 0.f;
  for (int i = threadIdx.x; i < PROW / 4; i += kThreads) reinterpret_cast<uint32_t*>(sZ)[i] = 0u;
  for (int r = threadIdx.x; r < kRows; r += kThreads) {
    float l = INFINITY;  // padding rows: p = 0
    if (r < rows) l = lse[(r % ph) * pw + x0 + r / ph];
    sL[r] = l;
  }
  {  // gathered query rows
    constexpr int CH = D / 8;
    for (int idx = threadIdx.x; idx < kRows * CH; idx += kThreads) {
      const int r = idx / CH, c = idx % CH;
      const bool ok = r < rows;
      const long long tok = ok ? static_cast<long long>(f) * P + (r % ph) * pw + x0 + r / ph : 0;
      cp_async16(sQ + swz(r, c, 2 * D), qh + tok * D + c * 8, ok);
    }
  }
  load_tile_async<D, kKeys, kThreads>(sK, k, 0, N);
  cp_async_commit();

  // this warp's 16 x 8 Gram blocks: b = w, w + 8, ... over (xl, mt, nt)
  const int MT = ceil_div(ph, 16), NT = ceil_div(ph, 8);
  const int nblk = nx * MT * NT;
  float acc[kMaxBlocks][4];
#pragma unroll
  for (int i = 0; i < kMaxBlocks; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;

  uint32_t qa[D / 16][4];
  const int n_stages = ceil_div(N, kKeys);
  for (int st = 0; st < n_stages; ++st) {
    if (st + 1 < n_stages) {
      load_tile_async<D, kKeys, kThreads>(sK + ((st + 1) & 1) * TILE, k, (st + 1) * kKeys, N);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    if (st == 0) load_a_frags<D>(qa, smem_u32(sQ), warp * 16);
    {  // probabilities of this warp's 16 rows for the stage's 64 keys
      float s[kKeys / 8][4];
      qk_frags<D, kKeys>(s, qa, smem_u32(sK + (st & 1) * TILE), 0);
      const int key0 = st * kKeys;
      const int ra = warp * 16 + g, rb = ra + 8;
      const float la = sL[ra], lb = sL[rb];
#pragma unroll
      for (int n = 0; n < kKeys / 8; ++n) {
        const int col = key0 + 8 * n + 2 * t4;
        const bool c0 = col < N, c1 = col + 1 < N;
        const float p0 = c0 ? fast_exp2(s[n][0] * a.scale_log2 - la) : 0.f;
        const float p1 = c1 ? fast_exp2(s[n][1] * a.scale_log2 - la) : 0.f;
        const float p2 = c0 ? fast_exp2(s[n][2] * a.scale_log2 - lb) : 0.f;
        const float p3 = c1 ? fast_exp2(s[n][3] * a.scale_log2 - lb) : 0.f;
        *reinterpret_cast<uint32_t*>(sP + ra * PROW + ((n ^ (ra & 7)) << 4) + 4 * t4) =
            pack_f16x2(p0, p1);
        *reinterpret_cast<uint32_t*>(sP + rb * PROW + ((n ^ (rb & 7)) << 4) + 4 * t4) =
            pack_f16x2(p2, p3);
      }
    }
    __syncthreads();
    // G += P_x P_x^T for this warp's blocks
#pragma unroll
    for (int i = 0; i < kMaxBlocks; ++i) {
      const int b = warp + 8 * i;
      if (b >= nblk) break;
      const int xl = b / (MT * NT), mt = (b / NT) % MT, nt = b % NT;
      const int ya = 16 * mt + (lane & 15);
      const int yb = 8 * nt + (lane & 7);
      const int rA = xl * ph + ya, rB = xl * ph + yb;
#pragma unroll
      for (int kk = 0; kk < kKeys / 16; ++kk) {
        const int ca = 2 * kk + (lane >> 4);
        const int cb = 2 * kk + ((lane >> 3) & 1);
        const uint32_t pa = ya < ph ? smem_u32(sP + rA * PROW + ((ca ^ (rA & 7)) << 4))
                                    : smem_u32(sZ + (ca << 4));
        const uint32_t pb = yb < ph ? smem_u32(sP + rB * PROW + ((cb ^ (rB & 7)) << 4))
                                    : smem_u32(sZ + (cb << 4));
        uint32_t fa[4], fb[2];
        ldmatrix_x4(fa[0], fa[1], fa[2], fa[3], pa);
        ldmatrix_x2(fb[0], fb[1], pb);
        mma_f16_16816(acc[i], fa, fb);
      }
    }
    __syncthreads();
  }
  // sum the column groups' blocks into the upper triangle
#pragma unroll
  for (int i = 0; i < kMaxBlocks; ++i) {
    const int b = warp + 8 * i;
    if (b >= nblk) break;
    const int mt = (b / NT) % MT, nt = b % NT;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int y = 16 * mt + g + 8 * (e >> 1), y2 = 8 * nt + 2 * t4 + (e & 1);
      if (y < ph && y2 < ph && y <= y2) atomicAdd(&sG[tri_index(y, y2, ph)], acc[i][e]);
    }
  }
  __syncthreads();
  float* out = a.gram + ((static_cast<long long>(bh) * a.nf + fi) * a.ng + grp) * tri;
  for (int i = threadIdx.x; i < tri; i += kThreads) out[i] = sG[i];
}

// fp32 inputs: SIMT, one column per CTA (gx = 1); tile row r = y.
template <int D>
__global__ void __launch_bounds__(128) rs_lse_fp32(const RsArgs a) {
  const int r = blockIdx.x * 128 + threadIdx.x, fi = blockIdx.y, bh = blockIdx.z;
  const int f = eval_frame(a.frames, fi, a.F, a.status);
  if (r >= a.P) return;
  const int N = a.N;
  const float* q = static_cast<const float*>(a.q) +
                   (static_cast<long long>(bh) * N + static_cast<long long>(f) * a.P + r) * D;
  const float* k = static_cast<const float*>(a.k) + static_cast<long long>(bh) * N * D;
  float m = -INFINITY, l = 0.f;
  for (int j = 0; j < N; ++j) {
    float dot = 0.f;
    for (int e = 0; e < D; ++e) dot = fmaf(q[e], k[static_cast<long long>(j) * D + e], dot);
    const float t = dot * a.scale_log2;
    const float mn = fmaxf(m, t);
    l = l * exp2f(m - mn) + exp2f(t - mn);
    m = mn;
  }
  a.lse[(static_cast<long long>(bh) * a.nf + fi) * a.P + r] = m + log2f(l);
}

template <int D>
__global__ void __launch_bounds__(128) rs_gram_fp32(const RsArgs a) {
  extern __shared__ float fsm[];
  const int x = blockIdx.x, fi = blockIdx.y, bh = blockIdx.z;
  const int f = eval_frame(a.frames, fi, a.F, a.status);
  const int N = a.N, ph = a.ph, pw = a.pw, P = a.P;
  const int tri = ph * (ph + 1) / 2;
  float* sP = fsm;              // [ph][kKeys]
  float* sG = sP + ph * kKeys;  // [tri]
  for (int i = threadIdx.x; i < tri; i += blockDim.x) sG[i] = 0.f;
  const float* k = static_cast<const float*>(a.k) + static_cast<long long>(bh) * N * D;
  const float* lse = a.lse + (static_cast<long long>(bh) * a.nf + fi) * P;
  for (int key0 = 0; key0 < N; key0 += kKeys) {
    __syncthreads();
    for (int idx = threadIdx.x; idx < ph * kKeys; idx += blockDim.x) {
      const int y = idx / kKeys, j = key0 + idx % kKeys;
      float p = 0.f;
      if (j < N) {
        const float* q = static_cast<const float*>(a.q) +
                         (static_cast<long long>(bh) * N + static_cast<long long>(f) * P +
                          y * pw + x) * D;
        float dot = 0.f;
        for (int e = 0; e < D; ++e) dot = fmaf(q[e], k[static_cast<long long>(j) * D + e], dot);
        p = exp2f(dot * a.scale_log2 - lse[y * pw + x]);
      }
      sP[idx] = p;
    }
    __syncthreads();
    for (int t = threadIdx.x; t < tri; t += blockDim.x) {
      int y = 0, rem = t;
      while (rem >= ph - y) {
        rem -= ph - y;
        ++y;
      }
      const int y2 = y + rem;
      float s = 0.f;
      for (int j = 0; j < kKeys; ++j) s = fmaf(sP[y * kKeys + j], sP[y2 * kKeys + j], s);
      sG[t] += s;
    }
  }
  __syncthreads();
  float* out = a.gram + ((static_cast<long long>(bh) * a.nf + fi) * a.ng + x) * tri;
  for (int i = threadIdx.x; i < tri; i += blockDim.x) out[i] = sG[i];
}

// Cosines from the summed Gram matrices; mean over pairs, then frames.
__global__ void __launch_bounds__(kThreads) rs_finalize(const RsArgs a) {
  __shared__ float red[kThreads / 32];
  const int bh = blockIdx.x, ph = a.ph, tri = ph * (ph + 1) / 2;
  const int pairs = ph * (ph - 1) / 2;
  float total = 0.f;
  for (int fi = 0; fi < a.nf; ++fi) {
    const float* gm = a.gram + (static_cast<long long>(bh) * a.nf + fi) * a.ng * tri;
    auto G = [&](int y, int y2) {
      float s = 0.f;
      for (int g = 0; g < a.ng; ++g) s += gm[static_cast<long long>(g) * tri + tri_index(y, y2, ph)];
      return s;
    };
    float part = 0.f;
    for (int t = threadIdx.x; t < pairs; t += kThreads) {
      int y = 0, rem = t;  // t-th pair (y < y2) in row-major order
      while (rem >= ph - 1 - y) {
        rem -= ph - 1 - y;
        ++y;
      }
      const int y2 = y + 1 + rem;
      part += G(y, y2) * rsqrtf(G(y, y) * G(y2, y2));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = part;
    __syncthreads();
    if (threadIdx.x == 0) {
      float s = 0.f;
      for (int w = 0; w < kThreads / 32; ++w) s += red[w];
      total += s / static_cast<float>(pairs);
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) a.sim[bh] = total / static_cast<float>(a.nf);
}

size_t gram_smem_bf16(int D, int ph) {
  return static_cast<size_t>(kRows) * D * 2 + 2 * static_cast<size_t>(kKeys) * D * 2 +
         static_cast<size_t>(kRows) * kKeys * 2 + kKeys * 2 + kRows * 4 +
         static_cast<size_t>(ph) * (ph + 1) / 2 * 4;
}

size_t rs_workspace(int B, int H, int ph, int pw, int n_frames, int dtype) {
  const int P = ph * pw;
  const int gx = dtype == SVG_BF16 ? kRows / ph : 1;
  const int ng = ceil_div(pw, gx);
  const size_t lse = static_cast<size_t>(B) * H * n_frames * P * 4;
  const size_t gram = static_cast<size_t>(B) * H * n_frames * ng * (ph * (ph + 1) / 2) * 4;
  return (lse + 255) / 256 * 256 + (gram + 255) / 256 * 256;
}

template <int D>
svg_status launch_rs(RsArgs& a, int BH, int dtype, cudaStream_t s) {
  if (dtype == SVG_BF16) {
    const size_t lse_smem = static_cast<size_t>(kRows) * D * 2 + 2 * static_cast<size_t>(kKeys) * D * 2;
    const size_t gsmem = gram_smem_bf16(D, a.ph);
    if (cudaFuncSetAttribute(rs_lse_bf16<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(lse_smem)) != cudaSuccess ||
        cudaFuncSetAttribute(rs_gram_bf16<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(gsmem)) != cudaSuccess)
      return fail(SVG_ERR_CUDA, "row_similarity: cannot reserve shared memory");
    rs_lse_bf16<D><<<dim3(ceil_div(a.P, kRows), a.nf, BH), kThreads, lse_smem, s>>>(a);
    if (svg_status st = check_launch("row_similarity lse")) return st;
    rs_gram_bf16<D><<<dim3(a.ng, a.nf, BH), kThreads, gsmem, s>>>(a);
    if (svg_status st = check_launch("row_similarity gram")) return st;
  } else {
    const size_t gsmem = (static_cast<size_t>(a.ph) * kKeys + a.ph * (a.ph + 1) / 2) * 4;
    if (gsmem > 48 * 1024)
      return fail(SVG_ERR_UNSUPPORTED, "row_similarity: ph=%d too large for fp32", a.ph);
    rs_lse_fp32<D><<<dim3(ceil_div(a.P, 128), a.nf, BH), 128, 0, s>>>(a);
    if (svg_status st = check_launch("row_similarity lse")) return st;
    rs_gram_fp32<D><<<dim3(a.ng, a.nf, BH), 128, gsmem, s>>>(a);
    if (svg_status st = check_launch("row_similarity gram")) return st;
  }
  rs_finalize<<<BH, kThreads, 0, s>>>(a);
  return check_launch("row_similarity finalize");
}

// --------------------------------------------------------------- anchor lists

// Does query tile i hold a token on an anchor row?  Image rows are runs of
// pw consecutive tokens starting at multiples of pw, so the tile is checked
// one row at a time.
__device__ bool tile_has_anchor(int i, int N, int P, int ph, int pw, int k) {
  const int lo = i * SVG_TILE, hi = min(N, lo + SVG_TILE);
  for (int n = lo; n < hi; n = (n / pw + 1) * pw) {
    const int y = (n % P) / pw;
    if (anchor_of(y, ph, k) == y) return true;
  }
  return false;
}

struct AnchorArgs {
  const int32_t* indptr;
  const int32_t* indices;
  int32_t* out_indptr;
  int32_t* out_indices;
  long long capacity;
  int n_lists, nqb, N, P, ph, pw, k;
  int32_t* status;
};

// One CTA: entries kept per (list copy, tile) row, then their exclusive scan
// into the output CSR (list copy c < n_lists is list c unchanged, copy
// n_lists + c is list c with anchor-free tiles emptied).
__global__ void __launch_bounds__(1024) anchor_scan_kernel(const AnchorArgs a) {
  __shared__ long long part[1024];
  __shared__ long long carry;
  const int R = 2 * a.n_lists * a.nqb;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < R; base += 1024) {
    const int row = base + threadIdx.x;
    long long cnt = 0;
    if (row < R) {
      const int copy = row / a.nqb, i = row % a.nqb;
      const int l = copy % a.n_lists;
      const int b = a.indptr[l * (a.nqb + 1) + i], e = a.indptr[l * (a.nqb + 1) + i + 1];
      if (b < 0 || e < b) {
        set_status(a.status, SVG_DEVICE_BAD_INDEX);
      } else if (copy < a.n_lists || tile_has_anchor(i, a.N, a.P, a.ph, a.pw, a.k)) {
        cnt = e - b;
      }
    }
    part[threadIdx.x] = cnt;
    __syncthreads();
    for (int off = 1; off < 1024; off <<= 1) {
      const long long y = threadIdx.x >= off ? part[threadIdx.x - off] : 0;
      __syncthreads();
      part[threadIdx.x] += y;
      __syncthreads();
    }
    if (row < R) {
      const int copy = row / a.nqb, i = row % a.nqb;
      const long long start = carry + part[threadIdx.x] - cnt;
      a.out_indptr[copy * (a.nqb + 1) + i] = static_cast<int32_t>(start);
      if (i == a.nqb - 1) a.out_indptr[copy * (a.nqb + 1) + a.nqb] = static_cast<int32_t>(start + cnt);
    }
    __syncthreads();
    if (threadIdx.x == 0) carry += part[1023];
    __syncthreads();
  }
  if (threadIdx.x == 0 && carry > a.capacity) set_status(a.status, SVG_DEVICE_CAPACITY);
}

// Warp per output row: copy the kept entries.
__global__ void __launch_bounds__(256) anchor_fill_kernel(const AnchorArgs a) {
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= 2 * a.n_lists * a.nqb) return;
  const int copy = row / a.nqb, i = row % a.nqb, l = copy % a.n_lists;
  const int o0 = a.out_indptr[copy * (a.nqb + 1) + i], o1 = a.out_indptr[copy * (a.nqb + 1) + i + 1];
  const int b = a.indptr[l * (a.nqb + 1) + i];
  for (int t = lane; t < o1 - o0; t += 32)
    if (o0 + t < a.capacity) a.out_indices[o0 + t] = a.indices[b + t];
}

// One CTA per output list: its pairing order.  Copies of the input lists
// keep index order; anchor copies put the tiles holding anchor rows first.
__global__ void __launch_bounds__(1024) anchor_order_kernel(const AnchorArgs a, int32_t* order) {
  __shared__ int part[1024];
  __shared__ int carry, n_live;
  const int copy = blockIdx.x, nqb = a.nqb;
  int32_t* out = order + static_cast<long long>(copy) * nqb;
  if (copy < a.n_lists) {
    for (int i = threadIdx.x; i < nqb; i += 1024) out[i] = i;
    return;
  }
  if (threadIdx.x == 0) {
    carry = 0;
    n_live = 0;
  }
  __syncthreads();
  int mine = 0;
  for (int i = threadIdx.x; i < nqb; i += 1024)
    mine += tile_has_anchor(i, a.N, a.P, a.ph, a.pw, a.k) ? 1 : 0;
  atomicAdd(&n_live, mine);
  __syncthreads();
  for (int base = 0; base < nqb; base += 1024) {
    const int i = base + threadIdx.x;
    const int live = (i < nqb && tile_has_anchor(i, a.N, a.P, a.ph, a.pw, a.k)) ? 1 : 0;
    part[threadIdx.x] = live;
    __syncthreads();
    for (int off = 1; off < 1024; off <<= 1) {
      const int y = threadIdx.x >= off ? part[threadIdx.x - off] : 0;
      __syncthreads();
      part[threadIdx.x] += y;
      __syncthreads();
    }
    if (i < nqb) {
      const int before = carry + part[threadIdx.x] - live;  // live tiles before i
      out[live ? before : n_live + (i - before)] = i;
    }
    __syncthreads();
    if (threadIdx.x == 0) carry += part[1023];
    __syncthreads();
  }
}

__global__ void anchor_ids_kernel(const int32_t* list_id, const int32_t* repeat, int n, int n_lists,
                                  int skip_list, int32_t* out) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const int l = list_id[i];
  const bool move = repeat != nullptr && repeat[i] != 0 && l >= 0 && l < n_lists && l != skip_list;
  out[i] = move ? l + n_lists : l;
}

// ------------------------------------------------------------------ broadcast

constexpr int kBcUnroll = 4;

__global__ void __launch_bounds__(256) broadcast_kernel(int4* __restrict__ o, int N, int chunk_log2,
                                                        int P, int ph, int pw, int k,
                                                        const int32_t* __restrict__ list_id,
                                                        int n_lists) {
  const int bh = blockIdx.y;
  if (list_id[bh] < n_lists) return;  // not a repeating head
  const long long head_chunks = static_cast<long long>(N) << chunk_log2;
  int4* oh = o + head_chunks * bh;
  const int cmask = (1 << chunk_log2) - 1;
  const long long base = static_cast<long long>(blockIdx.x) * (256 * kBcUnroll) + threadIdx.x;
  int4 v[kBcUnroll];
  long long dst[kBcUnroll];
#pragma unroll
  for (int i = 0; i < kBcUnroll; ++i) {
    const long long j = base + i * 256;
    dst[i] = -1;
    if (j < head_chunks) {
      const int n = static_cast<int>(j >> chunk_log2);
      const int f = n / P, s = n - f * P, y = s / pw;
      const int ay = anchor_of(y, ph, k);
      if (ay != y) {
        const long long src = static_cast<long long>(f) * P + ay * pw + (s - y * pw);
        v[i] = oh[(src << chunk_log2) | (static_cast<int>(j) & cmask)];
        dst[i] = j;
      }
    }
  }
#pragma unroll
  for (int i = 0; i < kBcUnroll; ++i)
    if (dst[i] >= 0) oh[dst[i]] = v[i];
}

}  // namespace
}  // namespace svg

using namespace svg;

namespace {

svg_status check_frame_shape(const char* who, int N, int F, int ph, int pw) {
  if (F <= 0 || ph <= 0 || pw <= 0 || static_cast<long long>(F) * ph * pw != N)
    return fail(SVG_ERR_INVALID_ARG, "%s: frames*rows*cols (%d*%d*%d) != N (%d)", who, F, ph, pw,
                N);
  return SVG_OK;
}

}  // namespace

extern "C" size_t svg_row_similarity_workspace_size(int dtype, int B, int H, int rows, int cols,
                                                    int n_frames) {
  if (B <= 0 || H <= 0 || rows <= 0 || cols <= 0 || n_frames <= 0) return 0;
  return rs_workspace(B, H, rows, cols, n_frames, dtype);
}

extern "C" svg_status svg_row_similarity(const void* q, const void* k, int dtype, int B, int H,
                                         int N, int d, int frames, int rows, int cols,
                                         const int32_t* eval_frames, int n_frames,
                                         float* sim_out, void* workspace, size_t workspace_bytes,
                                         int32_t* device_status, void* stream) {
  clear_error();
  if (q == nullptr || k == nullptr || sim_out == nullptr)
    return fail(SVG_ERR_INVALID_ARG, "row_similarity: null pointer");
  if (dtype != SVG_BF16 && dtype != SVG_FP32)
    return fail(SVG_ERR_INVALID_ARG, "row_similarity: bad dtype %d", dtype);
  if (B <= 0 || H <= 0 || N <= 0 || B * H > 65535)
    return fail(SVG_ERR_INVALID_ARG, "row_similarity: bad shape");
  if (d != 64 && d != 128)
    return fail(SVG_ERR_INVALID_ARG, "row_similarity: d=%d not in {64,128}", d);
  if (svg_status st = check_frame_shape("row_similarity", N, frames, rows, cols)) return st;
  if (rows < 2 || rows > kRows)
    return fail(SVG_ERR_INVALID_ARG, "row_similarity: rows=%d not in [2, %d]", rows, kRows);
  if (n_frames <= 0 || n_frames > 65535 || (eval_frames == nullptr && n_frames > frames))
    return fail(SVG_ERR_INVALID_ARG, "row_similarity: bad n_frames %d", n_frames);
  if (!aligned16(q) || !aligned16(k))
    return fail(SVG_ERR_INVALID_ARG, "row_similarity: tensors must be 16-byte aligned");
  if (dtype == SVG_BF16 &&
      (cols < kRows / rows ? cols : kRows / rows) * ceil_div(rows, 16) * ceil_div(rows, 8) >
          8 * kMaxBlocks)
    return fail(SVG_ERR_UNSUPPORTED, "row_similarity: rows=%d needs too many Gram blocks", rows);
  const size_t need = rs_workspace(B, H, rows, cols, n_frames, dtype);
  if (workspace == nullptr || !aligned256(workspace) || workspace_bytes < need)
    return fail(SVG_ERR_INVALID_ARG, "row_similarity: workspace too small or not 256-byte aligned");
  RsArgs a;
  a.q = q;
  a.k = k;
  a.frames = eval_frames;
  a.status = device_status;
  a.sim = sim_out;
  a.N = N;
  a.F = frames;
  a.ph = rows;
  a.pw = cols;
  a.P = rows * cols;
  a.nf = n_frames;
  a.gx = dtype == SVG_BF16 ? kRows / rows : 1;
  a.ng = ceil_div(cols, a.gx);
  const size_t lse_bytes = static_cast<size_t>(B) * H * n_frames * a.P * 4;
  a.lse = static_cast<float*>(workspace);
  a.gram = reinterpret_cast<float*>(static_cast<char*>(workspace) + (lse_bytes + 255) / 256 * 256);
  a.scale_log2 = kLog2e / sqrtf(static_cast<float>(d));
  cudaStream_t s = as_stream(stream);
  return d == 64 ? launch_rs<64>(a, B * H, dtype, s) : launch_rs<128>(a, B * H, dtype, s);
}

extern "C" svg_status svg_anchor_lists(int n_lists, int n_qblocks, const int32_t* indptr,
                                       const int32_t* indices, int N, int frames, int rows,
                                       int cols, int anchors, const int32_t* list_id,
                                       const int32_t* repeat, int n_heads, int skip_list,
                                       int32_t* out_indptr, int32_t* out_indices,
                                       int64_t capacity, int32_t* list_id_out,
                                       int32_t* tile_order_out, int32_t* device_status,
                                       void* stream) {
  clear_error();
  if (indptr == nullptr || indices == nullptr || out_indptr == nullptr ||
      out_indices == nullptr || (list_id != nullptr && list_id_out == nullptr))
    return fail(SVG_ERR_INVALID_ARG, "anchor_lists: null pointer");
  if (n_lists <= 0 || (list_id != nullptr && n_heads <= 0) || N <= 0 ||
      n_qblocks != n_tiles(N))
    return fail(SVG_ERR_INVALID_ARG, "anchor_lists: bad sizes (n_qblocks must be ceil(N/128))");
  if (static_cast<long long>(2) * n_lists * n_qblocks > 0x7fffffffLL)
    return fail(SVG_ERR_INVALID_ARG, "anchor_lists: too many rows");
  if (svg_status st = check_frame_shape("anchor_lists", N, frames, rows, cols)) return st;
  if (anchors <= 0) return fail(SVG_ERR_INVALID_ARG, "anchor_lists: anchors must be >= 1");
  if (capacity <= 0) return fail(SVG_ERR_INVALID_ARG, "anchor_lists: capacity must be > 0");
  AnchorArgs a;
  a.indptr = indptr;
  a.indices = indices;
  a.out_indptr = out_indptr;
  a.out_indices = out_indices;
  a.capacity = capacity;
  a.n_lists = n_lists;
  a.nqb = n_qblocks;
  a.N = N;
  a.P = rows * cols;
  a.ph = rows;
  a.pw = cols;
  a.k = anchors;
  a.status = device_status;
  cudaStream_t s = as_stream(stream);
  anchor_scan_kernel<<<1, 1024, 0, s>>>(a);
  if (svg_status st = check_launch("anchor_lists scan")) return st;
  const int R = 2 * n_lists * n_qblocks;
  anchor_fill_kernel<<<ceil_div(R, 8), 256, 0, s>>>(a);
  if (svg_status st = check_launch("anchor_lists fill")) return st;
  if (tile_order_out != nullptr) {
    anchor_order_kernel<<<2 * n_lists, 1024, 0, s>>>(a, tile_order_out);
    if (svg_status st = check_launch("anchor_lists order")) return st;
  }
  if (list_id == nullptr) return SVG_OK;  // lists only
  anchor_ids_kernel<<<ceil_div(n_heads, 256), 256, 0, s>>>(list_id, repeat, n_heads, n_lists,
                                                          skip_list, list_id_out);
  return check_launch("anchor_lists ids");
}

extern "C" svg_status svg_anchor_list_ids(const int32_t* list_id, const int32_t* repeat,
                                          int n_heads, int n_lists, int skip_list,
                                          int32_t* list_id_out, void* stream) {
  clear_error();
  if (list_id == nullptr || list_id_out == nullptr)
    return fail(SVG_ERR_INVALID_ARG, "anchor_list_ids: null pointer");
  if (n_heads <= 0 || n_lists <= 0)
    return fail(SVG_ERR_INVALID_ARG, "anchor_list_ids: bad sizes");
  anchor_ids_kernel<<<ceil_div(n_heads, 256), 256, 0, as_stream(stream)>>>(
      list_id, repeat, n_heads, n_lists, skip_list, list_id_out);
  return check_launch("anchor_list_ids");
}

extern "C" svg_status svg_row_broadcast(void* o, int dtype, int B, int H, int N, int d, int frames,
                                        int rows, int cols, int anchors, const int32_t* list_id,
                                        int n_lists, void* stream) {
  clear_error();
  if (o == nullptr || list_id == nullptr)
    return fail(SVG_ERR_INVALID_ARG, "row_broadcast: null pointer");
  if (dtype != SVG_BF16 && dtype != SVG_FP32)
    return fail(SVG_ERR_INVALID_ARG, "row_broadcast: bad dtype %d", dtype);
  if (B <= 0 || H <= 0 || N <= 0 || B * H > 65535)
    return fail(SVG_ERR_INVALID_ARG, "row_broadcast: bad shape");
  if (d != 64 && d != 128) return fail(SVG_ERR_INVALID_ARG, "row_broadcast: d=%d not in {64,128}", d);
  if (svg_status st = check_frame_shape("row_broadcast", N, frames, rows, cols)) return st;
  if (anchors <= 0 || n_lists <= 0)
    return fail(SVG_ERR_INVALID_ARG, "row_broadcast: anchors and n_lists must be >= 1");
  if (!aligned16(o)) return fail(SVG_ERR_INVALID_ARG, "row_broadcast: o must be 16-byte aligned");
  const int row_chunks = d * elt_bytes(dtype) / 16;
  int chunk_log2 = 0;
  while ((1 << chunk_log2) < row_chunks) ++chunk_log2;
  const long long blocks = (static_cast<long long>(N) * row_chunks + 256 * kBcUnroll - 1) /
                           (256 * kBcUnroll);
  if (blocks > 0x7fffffffLL) return fail(SVG_ERR_INVALID_ARG, "row_broadcast: N too large");
  broadcast_kernel<<<dim3(static_cast<unsigned>(blocks), B * H), 256, 0, as_stream(stream)>>>(
      static_cast<int4*>(o), N, chunk_log2, rows * cols, rows, cols, anchors, list_id, n_lists);
  return check_launch("row_broadcast");
}
