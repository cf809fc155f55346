// Arguments shared by the block-sparse attention kernels.
#pragma once

#include "common.cuh"

namespace svg {

struct AttnArgs {
  const void* q;
  const void* k;
  const void* v;
  void* o;
  int dtype;
  int B, H, N, d;
  const int32_t* list_id;  // [B*H]
  int n_lists, n_qblocks;
  const int32_t* indptr;   // [n_lists][n_qblocks + 1]
  const int32_t* indices;
  float scale;
  int32_t* status;         // optional device status word
  // Optional fused layout transformation for heads whose order[b*H + h] is
  // SVG_MODE_TEMPORAL (they run in token-major order, m = s * F + f):
  // SVG_FUSE_INPUT  q, k, v of such heads are frame-major in memory
  //                 (n = f * P + s) and gathered row by row;
  // SVG_FUSE_OUTPUT o of such heads is written frame-major.
  // order == nullptr or layout == 0: every tensor is in the heads' order.
  const int32_t* order;
  int frames, tokens_per_frame;
  int layout;
  // Optional token-major copies of q, k, v (every head reordered, e.g. by
  // svg_permute_token_major with no mode): heads whose order is
  // SVG_MODE_TEMPORAL read these, the others read q, k, v.  Set together or
  // not at all; exclusive with SVG_FUSE_INPUT.
  const void* q_tm;
  const void* k_tm;
  const void* v_tm;
  // Optional [n_lists][n_qblocks] pairing order: the tcgen05 kernel takes
  // the query tiles of a head two at a time in this order (a permutation of
  // 0 .. n_qblocks-1 per list); null = index order.  Results never depend
  // on it.
  const int32_t* tile_order;
  // Optional per-(b, h) V exponents from svg_v_exponents: the tcgen05 kernel
  // converts v * 2^-e to fp16 and multiplies the head's output by 2^e (a
  // value of 255 marks inf / NaN: converted unscaled).  Null: e = 0.
  const int32_t* v_exp;
  // Polls of one mbarrier wait before the tcgen05 kernel gives up with
  // SVG_DEVICE_TIMEOUT (svg_set_wait_limit).
  uint32_t spin_limit;
};

__device__ __forceinline__ bool reads_copies(const AttnArgs& a, int bh);

__device__ __forceinline__ bool temporal_head(const AttnArgs& a, int bh) {
  return a.order != nullptr && a.order[bh] == SVG_MODE_TEMPORAL;
}
__device__ __forceinline__ bool gathers_input(const AttnArgs& a, int bh) {
  return (a.layout & SVG_FUSE_INPUT) != 0 && temporal_head(a, bh);
}
__device__ __forceinline__ bool scatters_output(const AttnArgs& a, int bh) {
  return (a.layout & SVG_FUSE_OUTPUT) != 0 && temporal_head(a, bh);
}
__device__ __forceinline__ bool reads_copies(const AttnArgs& a, int bh) {
  return a.q_tm != nullptr && temporal_head(a, bh);
}

// Query tile in pairing slot `slot` of head bh (the list's tile order, or
// the slot itself); -1 past the end or for an out-of-range order entry.
__device__ __forceinline__ int query_tile(const AttnArgs& a, int bh, int slot, int nb) {
  if (slot >= nb) return -1;
  if (a.tile_order == nullptr) return slot;
  const int lid = a.list_id[bh];
  if (lid < 0 || lid >= a.n_lists) return slot;  // the list walk reports the bad id
  const int qt = a.tile_order[static_cast<long long>(lid) * a.n_qblocks + slot];
  return (qt >= 0 && qt < nb) ? qt : -1;
}

// Frame-major memory row of token-major row m.
__device__ __forceinline__ int token_major_row(int m, int F, int P) { return (m % F) * P + m / F; }

template <int D>
svg_status launch_attn_fp32(const AttnArgs& a, cudaStream_t s);
template <int D>
svg_status launch_attn_sm100(const AttnArgs& a, cudaStream_t s);

}  // namespace svg
