// svg_sparse_attn: argument validation and dispatch.
#include <math.h>

#include "attn.cuh"

using namespace svg;

namespace {

svg_status sparse_attn_impl(const char* who, const void* q, const void* k, const void* v, void* o,
                            int dtype, int B, int H, int N, int d, const int32_t* list_id,
                            int n_lists, int n_qblocks, const int32_t* indptr,
                            const int32_t* indices, float scale, int32_t* device_status,
                            const int32_t* order, int frames, int tokens_per_frame, int layout,
                            const void* q_tm, const void* k_tm, const void* v_tm,
                            const int32_t* tile_order, const int32_t* v_exp, void* stream) {
  clear_error();
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr || list_id == nullptr ||
      indptr == nullptr || indices == nullptr)
    return fail(SVG_ERR_INVALID_ARG, "%s: null pointer", who);
  if (dtype != SVG_BF16 && dtype != SVG_FP32)
    return fail(SVG_ERR_INVALID_ARG, "%s: bad dtype %d", who, dtype);
  if (B <= 0 || H <= 0 || N <= 0 || B * H > 65535)
    return fail(SVG_ERR_INVALID_ARG, "%s: bad shape B=%d H=%d N=%d", who, B, H, N);
  if (d != 64 && d != 128) return fail(SVG_ERR_INVALID_ARG, "%s: d=%d not in {64,128}", who, d);
  if (n_lists <= 0) return fail(SVG_ERR_INVALID_ARG, "%s: n_lists must be positive", who);
  if (n_qblocks != n_tiles(N))
    return fail(SVG_ERR_INVALID_ARG, "%s: n_qblocks=%d but ceil(N/128)=%d", who, n_qblocks,
                n_tiles(N));
  if ((layout & ~(SVG_FUSE_INPUT | SVG_FUSE_OUTPUT)) != 0)
    return fail(SVG_ERR_INVALID_ARG, "%s: bad layout %d", who, layout);
  if (order != nullptr && layout != 0 &&
      (frames <= 0 || tokens_per_frame <= 0 ||
       static_cast<long long>(frames) * tokens_per_frame != N))
    return fail(SVG_ERR_INVALID_ARG, "%s: frames * tokens_per_frame must equal N", who);
  const bool copies = q_tm != nullptr || k_tm != nullptr || v_tm != nullptr;
  if (copies && (q_tm == nullptr || k_tm == nullptr || v_tm == nullptr))
    return fail(SVG_ERR_INVALID_ARG, "%s: give all three token-major copies or none", who);
  if (copies && (layout & SVG_FUSE_INPUT) != 0)
    return fail(SVG_ERR_INVALID_ARG, "%s: token-major copies exclude SVG_FUSE_INPUT", who);
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      (copies && (!aligned16(q_tm) || !aligned16(k_tm) || !aligned16(v_tm))))
    return fail(SVG_ERR_INVALID_ARG, "%s: tensors must be 16-byte aligned", who);
  const long long bytes = static_cast<long long>(B) * H * N * d * elt_bytes(dtype);
  const char* ob = static_cast<const char*>(o);
  for (const void* t : {q, k, v, q_tm, k_tm, v_tm}) {
    if (t == nullptr) continue;
    const char* tb = static_cast<const char*>(t);
    if (ob < tb + bytes && tb < ob + bytes)
      return fail(SVG_ERR_INVALID_ARG, "%s: o overlaps an input", who);
  }
  if (!(scale >= 0.f) || isinf(scale)) return fail(SVG_ERR_INVALID_ARG, "%s: bad scale", who);
  AttnArgs a{q, k, v, o, dtype, B, H, N, d, list_id, n_lists, n_qblocks, indptr, indices,
             scale == 0.f ? 1.f / sqrtf(static_cast<float>(d)) : scale, device_status,
             order, frames, tokens_per_frame, layout, q_tm, k_tm, v_tm, tile_order, v_exp,
             wait_limit()};
  cudaStream_t s = as_stream(stream);
  if (dtype == SVG_FP32) return d == 64 ? launch_attn_fp32<64>(a, s) : launch_attn_fp32<128>(a, s);
  return d == 64 ? launch_attn_sm100<64>(a, s) : launch_attn_sm100<128>(a, s);
}

}  // namespace

extern "C" svg_status svg_sparse_attn(const void* q, const void* k, const void* v, void* o,
                                      int dtype, int B, int H, int N, int d,
                                      const int32_t* list_id, int n_lists, int n_qblocks,
                                      const int32_t* indptr, const int32_t* indices, float scale,
                                      int32_t* device_status, const int32_t* v_exp,
                                      void* stream) {
  return sparse_attn_impl("sparse_attn", q, k, v, o, dtype, B, H, N, d, list_id, n_lists,
                          n_qblocks, indptr, indices, scale, device_status, nullptr, 0, 0, 0,
                          nullptr, nullptr, nullptr, nullptr, v_exp, stream);
}

extern "C" svg_status svg_sparse_attn_fused(const void* q, const void* k, const void* v,
                                            const void* q_tm, const void* k_tm,
                                            const void* v_tm, void* o, int dtype, int B, int H,
                                            int N, int d, int frames, int tokens_per_frame,
                                            const int32_t* mode, int layout, int n_lists,
                                            int n_qblocks, const int32_t* indptr,
                                            const int32_t* indices, const int32_t* tile_order,
                                            float scale, int32_t* device_status,
                                            const int32_t* v_exp, void* stream) {
  return sparse_attn_impl("sparse_attn_fused", q, k, v, o, dtype, B, H, N, d, mode, n_lists,
                          n_qblocks, indptr, indices, scale, device_status, mode, frames,
                          tokens_per_frame, layout, q_tm, k_tm, v_tm, tile_order, v_exp, stream);
}
