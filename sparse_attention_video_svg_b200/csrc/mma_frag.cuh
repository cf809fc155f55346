// Warp-level bf16 tensor-core fragments (mma.sync m16n8k16) over swizzled
// shared-memory tiles.  Used by the profiling and block-energy kernels, whose
// contractions have M = 64 sampled rows or stream every key tile once; the
// block-sparse attention kernel itself runs on tcgen05 (attn_sm100.cu).
//
// Tile layout: row r of a [rows][D] bf16 tile starts at r * 2D bytes; its
// 16-byte chunk c sits at chunk position c ^ (r & 7) (see swz()).
#pragma once

#include "common.cuh"

namespace svg {

// A fragments of the 16 x D query block at rows [row0, row0 + 16).
template <int D>
__device__ __forceinline__ void load_a_frags(uint32_t (&a)[D / 16][4], uint32_t tile, int row0) {
  const int lane = threadIdx.x & 31;
  const int r = row0 + (lane & 15);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const int c = 2 * kk + (lane >> 4);
    ldmatrix_x4(a[kk][0], a[kk][1], a[kk][2], a[kk][3], tile + swz(r, c, 2 * D));
  }
}

// s[n][.] = Q(16 x D) . K^T for the NK keys at rows [key0, key0 + NK) of the
// K tile (NK a multiple of 16).  Accumulator layout: s[n] covers keys
// key0 + 8n .. 8n + 7; s[n][0..1] row g, s[n][2..3] row g + 8, cols 2t, 2t+1.
template <int D, int NK>
__device__ __forceinline__ void qk_frags(float (&s)[NK / 8][4], const uint32_t (&a)[D / 16][4],
                                         uint32_t ktile, int key0) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int n = 0; n < NK / 8; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
  // K-steps outer, key groups inner: consecutive MMAs accumulate into
  // different s[n], so they pipeline (each s[n] still sums its K-steps in
  // order)
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const int c = 2 * kk + ((lane >> 3) & 1);
#pragma unroll
    for (int np = 0; np < NK / 16; ++np) {
      const int r = key0 + np * 16 + (lane & 7) + ((lane >> 4) << 3);
      uint32_t b0, b1, b2, b3;
      ldmatrix_x4(b0, b1, b2, b3, ktile + swz(r, c, 2 * D));
      const uint32_t bA[2] = {b0, b1};
      const uint32_t bB[2] = {b2, b3};
      mma_bf16_16816(s[2 * np], a[kk], bA);
      mma_bf16_16816(s[2 * np + 1], a[kk], bB);
    }
  }
}

// o += P(16 x NK) . V[key0 .. key0 + NK), P given as fp32 accumulator-layout
// values and rounded to bf16 here.
template <int D, int NK>
__device__ __forceinline__ void pv_frags(float (&o)[D / 8][4], const float (&p)[NK / 8][4],
                                         uint32_t vtile, int key0) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int kk = 0; kk < NK / 16; ++kk) {
    uint32_t a[4];
    a[0] = pack_bf16x2(p[2 * kk][0], p[2 * kk][1]);
    a[1] = pack_bf16x2(p[2 * kk][2], p[2 * kk][3]);
    a[2] = pack_bf16x2(p[2 * kk + 1][0], p[2 * kk + 1][1]);
    a[3] = pack_bf16x2(p[2 * kk + 1][2], p[2 * kk + 1][3]);
    const int r = key0 + kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
#pragma unroll
    for (int nn = 0; nn < D / 8; nn += 2) {
      const int c = nn + (lane >> 4);
      uint32_t b0, b1, b2, b3;
      ldmatrix_x4_trans(b0, b1, b2, b3, vtile + swz(r, c, 2 * D));
      const uint32_t bA[2] = {b0, b1};
      const uint32_t bB[2] = {b2, b3};
      mma_bf16_16816(o[nn], a, bA);
      mma_bf16_16816(o[nn + 1], a, bB);
    }
  }
}

// Asynchronously copies rows [row0, row0 + ROWS) of a [n_rows][D] bf16 global
// matrix into a swizzled smem tile (rows at or beyond n_rows are zero-filled).
template <int D, int ROWS, int THREADS>
__device__ __forceinline__ void load_tile_async(void* smem_tile, const __nv_bfloat16* g, int row0,
                                                int n_rows) {
  constexpr int CH = D / 8;  // 16-byte chunks per row
  char* base = static_cast<char*>(smem_tile);
  for (int idx = threadIdx.x; idx < ROWS * CH; idx += THREADS) {
    const int r = idx / CH, c = idx % CH;
    const int gr = row0 + r;
    const bool ok = gr < n_rows;
    const __nv_bfloat16* src = g + static_cast<long long>(ok ? gr : 0) * D + c * 8;
    cp_async16(base + swz(r, c, 2 * D), src, ok);
  }
}

}  // namespace svg
