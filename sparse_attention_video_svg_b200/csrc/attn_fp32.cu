// Block-sparse attention for fp32 inputs (SIMT fp32 arithmetic).
//
// Video-diffusion acceleration survey (wmrh.cn/news/48564), section 2.1:
// o = softmax(Q K^T / sqrt(d_k)) V.  CalibAtt article (lpnh.cn/news/568491),
// sections 2.2 and 3.3: keep/skip decisions per 128 x 128 tile, walked
// through a per-row list of kept key blocks.  bf16 inputs run on the tcgen05
// kernel (attn_sm100.cu); this path keeps fp32 inputs in fp32.
#include "attn.cuh"
#include "common.cuh"

namespace svg {
namespace {

constexpr float kLog2e = 1.4426950408889634f;

// The list of query tile qt of head bh; entries are validated lazily.
struct RowList {
  const int32_t* idx;
  int len;
};

__device__ __forceinline__ RowList row_list(const AttnArgs& a, int bh, int qt) {
  const int lid = a.list_id[bh];
  if (lid < 0 || lid >= a.n_lists) {
    if (qt == 0) set_status(a.status, SVG_DEVICE_BAD_LIST_ID);
    return {nullptr, 0};
  }
  const int32_t* ip = a.indptr + static_cast<long long>(lid) * (a.n_qblocks + 1);
  const int beg = ip[qt], end = ip[qt + 1];
  if (end < beg || beg < 0) {
    set_status(a.status, SVG_DEVICE_BAD_INDEX);
    return {nullptr, 0};
  }
  return {a.indices + beg, end - beg};
}

// fp32 SIMT: one warp per query row at a time, lanes split the head dim.
template <int D>
__global__ void __launch_bounds__(256) attn_fp32(AttnArgs a) {
  constexpr int E = D / 32;
  const int qt = blockIdx.x, bh = blockIdx.y;
  const int N = a.N, nb = n_tiles(N);
  const long long head = static_cast<long long>(bh) * N * D;
  const bool copies = reads_copies(a, bh);
  auto* q = static_cast<const float*>(copies ? a.q_tm : a.q) + head;
  auto* k = static_cast<const float*>(copies ? a.k_tm : a.k) + head;
  auto* v = static_cast<const float*>(copies ? a.v_tm : a.v) + head;
  auto* o = static_cast<float*>(a.o) + head;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const RowList lst = row_list(a, bh, qt);
  const float scale_log2 = a.scale * kLog2e;
  const bool gin = gathers_input(a, bh), sout = scatters_output(a, bh);
  const int F = a.frames, P = a.tokens_per_frame;
  // memory row of sequence position x in the inputs
  auto row = [&](int x) -> long long { return gin ? token_major_row(x, F, P) : x; };
  for (int r = qt * SVG_TILE + warp; r < min(N, (qt + 1) * SVG_TILE); r += 8) {
    float qv[E], acc[E], m = -INFINITY, l = 0.f;
    const long long rq = row(r);
    const long long ro = sout ? token_major_row(r, F, P) : r;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      qv[e] = q[rq * D + lane + 32 * e];
      acc[e] = 0.f;
    }
    int last = -1;
    for (int t = 0; t < lst.len; ++t) {
      const int j = lst.idx[t];
      // rows must be strictly ascending: an out-of-range, repeated or
      // descending entry is skipped, so no key block is attended twice
      if (j < 0 || j >= nb || j <= last) {
        set_status(a.status, SVG_DEVICE_BAD_INDEX);
        continue;
      }
      last = j;
      for (int c = j * SVG_TILE; c < min(N, (j + 1) * SVG_TILE); ++c) {
        const long long rc = row(c);
        float dot = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) dot = fmaf(qv[e], k[rc * D + lane + 32 * e], dot);
#pragma unroll
        for (int o2 = 16; o2 > 0; o2 >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o2);
        const float tt = dot * scale_log2;
        const float mn = fmaxf(m, tt);
        const float alpha = exp2f(m - mn);
        const float p = exp2f(tt - mn);
        l = l * alpha + p;
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] = fmaf(p, v[rc * D + lane + 32 * e], acc[e] * alpha);
        m = mn;
      }
    }
    const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) o[ro * D + lane + 32 * e] = acc[e] * inv;
  }
}

}  // namespace

template <int D>
svg_status launch_attn_fp32(const AttnArgs& a, cudaStream_t s) {
  dim3 grid(n_tiles(a.N), a.B * a.H);
  attn_fp32<D><<<grid, 256, 0, s>>>(a);
  return check_launch("sparse_attn fp32");
}

template svg_status launch_attn_fp32<64>(const AttnArgs&, cudaStream_t);
template svg_status launch_attn_fp32<128>(const AttnArgs&, cudaStream_t);

}  // namespace svg
