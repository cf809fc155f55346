// Pairing order of query tiles for the block-sparse attention kernel.
//
// CalibAtt article (lpnh.cn/news/568491), sections 2.2 and 3.3: attention is
// computed on 128 x 128 tiles walked through per-query-block lists of kept
// key blocks.  The sm100 kernel runs two query tiles of a head as one work
// item and loads a key block kept by both only once, so it is fastest when
// the two tiles of an item keep the same blocks.  Adjacent tiles do for
// geometric lists and for most calibrated lists; for calibrated lists of
// heads that attend along the time axis they share few blocks (the tiles
// that do are a frame apart).  This pass computes, per list, an order of the
// query tiles in which consecutive pairs (2i, 2i + 1) share many blocks:
// greedily, the smallest unpaired tile takes the unpaired tile whose row has
// the most blocks in common with its own (ties: the smaller tile index).
// A scheduling choice only: the attention results do not depend on it.
//
// One CTA per list: the rows become bitmaps in the workspace, then each pick
// scores every unpaired tile against the chosen one (AND + popcount over the
// row's words) and takes the maximum with a block reduction.
#include "common.cuh"

namespace svg {
namespace {

constexpr int kPairThreads = 256;

__global__ void __launch_bounds__(kPairThreads) pair_tiles_kernel(
    const int32_t* __restrict__ indptr, const int32_t* __restrict__ indices, int nq, int nk,
    int words, uint32_t* __restrict__ bits_all, int32_t* __restrict__ order_all,
    int32_t* __restrict__ status) {
  const int l = blockIdx.x, tid = threadIdx.x;
  const int32_t* ip = indptr + static_cast<long long>(l) * (nq + 1);
  uint32_t* bits = bits_all + static_cast<long long>(l) * nq * words;
  int32_t* order = order_all + static_cast<long long>(l) * nq;
  extern __shared__ uint32_t sm[];
  uint32_t* a_bits = sm;                                            // [words]
  unsigned long long* red = reinterpret_cast<unsigned long long*>(a_bits + words + (words & 1));
  unsigned char* taken = reinterpret_cast<unsigned char*>(red + kPairThreads / 32 + 1);  // [nq]
  __shared__ int s_a;

  // rows as bitmaps (each thread writes only the words of its own rows)
  for (long long i = tid; i < static_cast<long long>(nq) * words; i += kPairThreads) bits[i] = 0u;
  for (int i = tid; i < nq; i += kPairThreads) taken[i] = 0;
  __syncthreads();
  for (int r = tid; r < nq; r += kPairThreads) {
    const int b = ip[r], e = ip[r + 1];
    if (b < 0 || e < b) {
      set_status(status, SVG_DEVICE_BAD_INDEX);
      continue;
    }
    for (int t = b; t < e; ++t) {
      const int c = indices[t];
      if (c >= 0 && c < nk)
        bits[static_cast<long long>(r) * words + (c >> 5)] |= 1u << (c & 31);
      else
        set_status(status, SVG_DEVICE_BAD_INDEX);
    }
  }
  __syncthreads();

  int next = 0, pos = 0;
  while (true) {
    if (tid == 0) {
      while (next < nq && taken[next]) ++next;
      s_a = next;
      if (next < nq) taken[next] = 1;
    }
    __syncthreads();
    const int a = s_a;
    if (a >= nq) break;
    for (int w = tid; w < words; w += kPairThreads) a_bits[w] = bits[static_cast<long long>(a) * words + w];
    __syncthreads();
    // key = (overlap + 1) << 32 | (0xffffffff - c): the largest key is the
    // largest overlap, then the smallest index; 0 = no candidate
    unsigned long long best = 0;
    for (int c = tid; c < nq; c += kPairThreads) {
      if (taken[c]) continue;
      const uint32_t* row = bits + static_cast<long long>(c) * words;
      unsigned ov = 0;
      for (int w = 0; w < words; ++w) ov += __popc(a_bits[w] & row[w]);
      const unsigned long long key = (static_cast<unsigned long long>(ov + 1) << 32) |
                                     (0xffffffffu - static_cast<unsigned>(c));
      best = key > best ? key : best;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const unsigned long long other = __shfl_xor_sync(0xffffffffu, best, o);
      best = other > best ? other : best;
    }
    if ((tid & 31) == 0) red[tid >> 5] = best;
    __syncthreads();
    if (tid == 0) {
      for (int w = 1; w < kPairThreads / 32; ++w) best = red[w] > best ? red[w] : best;
      order[pos++] = a;
      if (best != 0) {
        const int b = static_cast<int>(0xffffffffu - static_cast<unsigned>(best & 0xffffffffu));
        order[pos++] = b;
        taken[b] = 1;
      }
    }
    __syncthreads();
  }
}

size_t words_for(int nk) { return (static_cast<size_t>(nk) + 31) / 32; }

}  // namespace
}  // namespace svg

using namespace svg;

extern "C" size_t svg_pair_query_tiles_workspace_size(int n_lists, int n_qblocks, int n_kblocks) {
  if (n_lists <= 0 || n_qblocks <= 0 || n_kblocks <= 0) return 0;
  return static_cast<size_t>(n_lists) * n_qblocks * words_for(n_kblocks) * sizeof(uint32_t);
}

extern "C" svg_status svg_pair_query_tiles(const int32_t* indptr, const int32_t* indices,
                                           int n_lists, int n_qblocks, int n_kblocks,
                                           int32_t* tile_order, int32_t* device_status,
                                           void* workspace, size_t workspace_bytes,
                                           void* stream) {
  clear_error();
  if (indptr == nullptr || tile_order == nullptr || workspace == nullptr)
    return fail(SVG_ERR_INVALID_ARG, "pair_query_tiles: null pointer");
  if (n_lists <= 0 || n_qblocks <= 0 || n_kblocks <= 0 || n_lists > 65535)
    return fail(SVG_ERR_INVALID_ARG, "pair_query_tiles: bad sizes (lists %d, rows %d, blocks %d)",
                n_lists, n_qblocks, n_kblocks);
  const size_t words = words_for(n_kblocks);
  const size_t smem = (words + 1) * sizeof(uint32_t) + (kPairThreads / 32 + 1) * 8 + n_qblocks;
  if (smem > 48 * 1024)
    return fail(SVG_ERR_INVALID_ARG, "pair_query_tiles: %d rows of %d blocks exceed the pass's limit",
                n_qblocks, n_kblocks);
  const size_t need = svg_pair_query_tiles_workspace_size(n_lists, n_qblocks, n_kblocks);
  if (workspace_bytes < need)
    return fail(SVG_ERR_INVALID_ARG, "pair_query_tiles: workspace %zu bytes, need %zu",
                workspace_bytes, need);
  if ((reinterpret_cast<uintptr_t>(workspace) & 3u) != 0)
    return fail(SVG_ERR_INVALID_ARG, "pair_query_tiles: workspace must be 4-byte aligned");
  if (indices == nullptr) return fail(SVG_ERR_INVALID_ARG, "pair_query_tiles: null indices");
  pair_tiles_kernel<<<n_lists, kPairThreads, smem, as_stream(stream)>>>(
      indptr, indices, n_qblocks, n_kblocks, static_cast<int>(words),
      static_cast<uint32_t*>(workspace), tile_order, device_status);
  return check_launch("pair_query_tiles");
}
