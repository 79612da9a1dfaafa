// Parameters and helpers shared by the two grouped-GEMM kernels (one CTA per unit in
// ffn_gemm.cu, an SM pair per unit in ffn_gemm_pair.cu).
#pragma once

#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

struct FfnParams {
  const int32_t *mblk;     // row chunks {row_start, expert, live rows <= 256}
  const int32_t *meta;     // meta[2] = number of row chunks
  const uint32_t *flags;   // pool tile flags (streaming)
  int32_t *status;
  uint16_t *out;           // act (GEMM A) or ypool (GEMM Y)
  int64_t out_ld;          // elements per row of out
  int32_t K;               // reduction length
  int32_t n_blocks;        // weight-column blocks per row chunk
  int32_t col_step;        // weight columns per block
  int32_t col1_off;        // first column of accumulator 1 inside the block's weights
  int32_t n_out;           // output columns (I or H): masks a ragged last block
  int32_t n_out1;          // the same limit for accumulator 1's columns (SM-pair kernel)
  int32_t k_rows;          // rows per expert in the weight tensor map ([E*H, 2I] W1: H,
                           // [E*I, H] W2: I), whichever way the MMA reads them
  int32_t tile;            // pool tile rows
  int32_t streaming;
  int32_t *sched;          // {next unit ticket, CTAs done}: zero at launch, zeroed again at exit
  int32_t sched_group;     // clusters (pair kernel) or CTAs of all launches sharing sched;
                           // 0 = this launch's own
  int32_t packed;          // weights are moe_pack_weights tiles (one 16 KB box per tile)
  // packed tile index = e*pk_e + nb*pk_nb + rank*pk_v + j*pk_j + kb
  // (rank = CTA of an SM pair, j = accumulator)
  int32_t pk_e, pk_j, pk_nb, pk_v;
  uint64_t timeout_ns;
  // SwiGLU backward epilogue (mode 2): g at aux[p*aux_ld + n], u at aux[p*aux_ld + aux_off + n];
  // dg and du written to out at the same offsets
  const uint16_t *aux;
  int64_t aux_ld;
  int32_t aux_off;
  // mode 3 (GEMM A saving gate / up): out = [g | u], act = bf16(silu(g) u) to out2
  uint16_t *out2;
  int64_t out2_ld;
  // early combine (GEMM Y of the SM-pair kernel): once all units of a row chunk are stored
  // (chunk_cnt reaches both CTAs x the column blocks), tok_pending[t] of each live row's
  // token t = row_src[p] / k drops by one; at zero t + 1 goes to the ready queue
  // ready[0 .. T) (tail at ready[T + 1]); after their GEMM work the CTAs pop tokens (head
  // at ready[T]) and write comb_out[t] = bf16(sum_j topk_w[t, j] ypool[pool_row[t, j]]).
  const int32_t *row_src;
  const int32_t *pool_row;
  const float *topk_w;
  int32_t *chunk_cnt;      // per row chunk: units stored by both CTAs (zero at launch)
  int32_t *tok_pending;
  int32_t *ready;
  uint16_t *comb_out;
  int32_t T, k;
};

// Order of the grouped GEMMs' units. The units of one expert (its row chunks x the weight
// column blocks) take consecutive tickets; inside them, chunks are taken kChunkBlock at a
// time, and for each such block of chunks every column block in turn, so the units that
// read the same weight columns start close together and share them through L2. Returns the
// unit's chunk (index into the row-chunk table) and weight column block.
#ifndef MOE_CHUNK_BLOCK
#define MOE_CHUNK_BLOCK 16
#endif
constexpr int kChunkBlock = MOE_CHUNK_BLOCK;

__device__ __forceinline__ void unit_coords(const int32_t *mblk, int32_t u, int32_t n_blocks,
                                            int32_t &mb, int32_t &nb) {
  if (kChunkBlock == 1) {
    mb = u / n_blocks;
    nb = u % n_blocks;
    return;
  }
  const int32_t *m = mblk + kMblkInts * (u / n_blocks);  // a chunk of the same expert
  const int32_t first = m[3], n_ch = m[4];
  const int32_t local = u - n_blocks * first;
  const int32_t b = local / (n_blocks * kChunkBlock);
  const int32_t cb = min(kChunkBlock, n_ch - b * kChunkBlock);
  const int32_t li = local - b * n_blocks * kChunkBlock;
  nb = li / cb;
  mb = first + b * kChunkBlock + li % cb;
}

// 2^x on the MUFU (ex2.approx.ftz.f32).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Magic-constant reciprocal for d in [1, 2^100], on the FMA pipe only. A float's bit
// pattern read as an integer is 2^23 (log2(value) + 127 - s(m)), where s(m) = m - log2(1 + m)
// >= 0 is the error of reading the mantissa m linearly. Hence bits(1/d) is close to
// 2 * 127 * 2^23 - bits(d) = 0x7F000000 - bits(d), and subtracting a constant shift c
// 2^23 from 0x7F000000 centres the error: kRecipMagic = 0x7F000000 - c 2^23. The shift is
// the minimax one, chosen so that the largest relative error of the first estimate over a
// binade (the error repeats in every binade) is as small as possible: a scan of the
// constant gives 5.051% at 0x7EF311C2, and 0x7EF311C7 (c = 0.10102) is within 4e-7 of
// that optimum (the host test of the SiLU method repeats the scan). This is the same
// derivation as the well-known inverse-square-root bit trick, applied to the exponent -1.
// Two Newton-Raphson steps y <- y (2 - d y) square the relative error twice: below 1e-5
// (measured 6.5e-6), far under the bf16 rounding (3.9e-3) of the act values it feeds.
constexpr int32_t kRecipMagic = 0x7EF311C7;
__device__ __forceinline__ float recip_newton2(float d) {
  float y = __int_as_float(kRecipMagic - __float_as_int(d));
  y = y * fmaf(-d, y, 2.0f);
  y = y * fmaf(-d, y, 2.0f);
  return y;
}

// silu(g) * u = g u / (1 + e^-g): one MUFU operation (the exponential) per element,
// the reciprocal on the FMA pipe. e^-g is capped at 2^100 (g below -69), where silu(g)
// is below 1e-28 in magnitude.
__device__ __forceinline__ float silu_mul(float g, float u) {
  const float e = ex2_approx(fminf(g * -1.4426950408889634f, 100.0f));
  return g * u * recip_newton2(1.0f + e);
}

__device__ __forceinline__ uint16_t bf16_bits(float v) {
  __nv_bfloat16 b = __float2bfloat16_rn(v);
  return *reinterpret_cast<uint16_t *>(&b);
}

// Row-major bf16 matrix [outer, inner] as a 2-D TMA tensor map, box {64, box_outer},
// 128-byte swizzle (the canonical layout tcgen05 descriptors read). ffn_gemm.cu.
bool make_tmap(CUtensorMap *m, const void *base, uint64_t inner, uint64_t outer,
               uint32_t box_outer);
// The same with any box and a swizzle of 0, 64 or 128 bytes (the span of one swizzled row).
bool make_tmap_box(CUtensorMap *m, const void *base, uint64_t inner, uint64_t outer,
                   uint32_t box_inner, uint32_t box_outer, uint32_t swizzle_bytes);

// Pair-kernel launch (ffn_gemm_pair.cu): grid = 2 * clusters CTAs, clusters of two.
// mode 0: SwiGLU epilogue (GEMM A); 1: plain bf16 (GEMM Y, backward A, gate / up
// recompute); 2: SwiGLU backward (backward Y); 3: GEMM A that also stores g | u. a_kmajor: the weights are read K-major
// (rows of the tensor map are output columns: W2 for backward Y, W1 for backward A).
// early: GEMM Y (mode 1, MN-major) with the combine fused in (prm.row_src ... comb_out).
cudaError_t launch_ffn_pair(int mode, bool a_kmajor, const CUtensorMap &tw,
                            const CUtensorMap &tx, const FfnParams &prm, int clusters,
                            cudaStream_t st, bool early = false);
// Clusters of two of the pair kernel that fit on the device at once (0 on error).
int ffn_pair_max_clusters(int mode);

}  // namespace moe
