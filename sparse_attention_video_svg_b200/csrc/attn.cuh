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
};

template <int D>
svg_status launch_attn_fp32(const AttnArgs& a, cudaStream_t s);
template <int D>
svg_status launch_attn_sm100(const AttnArgs& a, cudaStream_t s);

}  // namespace svg
