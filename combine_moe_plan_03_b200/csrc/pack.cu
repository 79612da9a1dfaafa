// Weight prepack for the grouped GEMMs: a one-time copy of W1 / W2 into tiles of
// 64 k-rows x 128 columns, each tile 16 KB and contiguous, in the byte order the
// GEMM's shared-memory tile takes (two 64-column halves one after the other, each
// 64 rows of 128 bytes). A GEMM unit then streams one contiguous region of HBM per
// weight tile sequence instead of 128-byte pieces at the matrix's row pitch.
//
// Tile numbering (tile = 128 rows of 64 bf16 in the packed array):
//   W1p: tile ((e*2 + g)*NB1 + nb)*KB1 + kb, g = 0 gate / 1 up, NB1 = ceil(I/128),
//        KB1 = H/64; row r = c*64 + kr holds W1[e][kb*64 + kr][g*I + nb*128 + c*64 + 0..63]
//   W2p: tile (e*NB2 + nb)*KB2 + kb, NB2 = 2*ceil(H/256), KB2 = I/64;
//        row r holds W2[e][kb*64 + kr][nb*128 + c*64 + 0..63]
// Columns past I (W1) or H (W2) are zero.
#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

PackGeom pack_geom(const moe_shape &s) {
  PackGeom g;
  g.nb1 = (s.I + 127) / 128;
  g.kb1 = s.H / 64;
  g.nb2 = 2 * ((s.H + 255) / 256);
  g.kb2 = s.I / 64;
  g.tiles1 = (int64_t)s.E * 2 * g.nb1 * g.kb1;
  g.tiles2 = (int64_t)s.E * g.nb2 * g.kb2;
  return g;
}

// One block per tile: 128 threads copy its 128 rows of 128 bytes (8 x 16 B each).
__global__ void __launch_bounds__(128)
    pack_kernel(const uint16_t *__restrict__ W, uint16_t *__restrict__ Wp, int64_t tiles,
                int32_t groups_per_expert, int32_t nb, int32_t kb, int32_t ld, int32_t valid_cols,
                int32_t group_col_stride, int32_t rows_per_expert) {
  for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x) {
    const int32_t k_blk = (int32_t)(t % kb);
    const int64_t rest = t / kb;
    const int32_t n_blk = (int32_t)(rest % nb);
    const int64_t rest2 = rest / nb;
    const int32_t grp = (int32_t)(rest2 % groups_per_expert);
    const int64_t e = rest2 / groups_per_expert;
    uint4 *dst = reinterpret_cast<uint4 *>(Wp + t * 128 * 64);
    for (int v = threadIdx.x; v < 128 * 8; v += blockDim.x) {
      const int r = v >> 3, q = v & 7;
      const int c = r >> 6, kr = r & 63;
      const int32_t col = n_blk * 128 + c * 64;  // column inside this group's columns
      uint4 val = make_uint4(0u, 0u, 0u, 0u);
      if (col < valid_cols) {
        const int64_t row = e * rows_per_expert + (int64_t)k_blk * 64 + kr;
        const uint4 *src = reinterpret_cast<const uint4 *>(
            W + row * ld + (int64_t)grp * group_col_stride + col);
        val = src[q];
      }
      dst[v] = val;
    }
  }
}

cudaError_t launch_pack(const moe_shape &s, const void *W1, const void *W2, void *W1p, void *W2p,
                        int num_sms, cudaStream_t st) {
  const PackGeom g = pack_geom(s);
  const int grid = num_sms * 16;
  if (g.tiles1 > 0) {
    pack_kernel<<<(int)(g.tiles1 < grid ? g.tiles1 : grid), 128, 0, st>>>(
        static_cast<const uint16_t *>(W1), static_cast<uint16_t *>(W1p), g.tiles1, 2, g.nb1,
        g.kb1, 2 * s.I, s.I, s.I, s.H);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (g.tiles2 > 0) {
    pack_kernel<<<(int)(g.tiles2 < grid ? g.tiles2 : grid), 128, 0, st>>>(
        static_cast<const uint16_t *>(W2), static_cast<uint16_t *>(W2p), g.tiles2, 1, g.nb2,
        g.kb2, s.H, s.H, 0, s.I);
    return cudaGetLastError();
  }
  return cudaSuccess;
}

}  // namespace moe
