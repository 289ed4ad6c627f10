// Internal definitions of the backward (gradient) kernels.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace flare {

constexpr int kBwdTokTile = 64;     // tokens per shared-memory tile of the latent-parallel kernels
constexpr int kBwdTokBlock = 128;   // tokens per CTA of the token-parallel kernels
// Latents per shared-memory chunk of the token-parallel kernels (two
// buffers of three [chunk][D + 4] fp32 operands stay within 48 KB).
__host__ __device__ constexpr int tok_chunk(int D) { return D == 16 ? 64 : 32; }
constexpr int kBwdDwRows = 2048;    // token rows per split of the weight-gradient GEMM

// Modes of the latent-parallel kernel (one CTA = a block of latents of one
// head and one token split; a warp = one or two tiles of 16 latent rows).
enum LatMode : int {
  kLatForward = 0,   // encoder recompute: per split (max, sum, sum w v) in log2 units
  kLatDecoder = 1,   // decoder backward, reductions over tokens: dZ and dQ
  kLatEncoder = 2,   // encoder backward, reduction over tokens: dQ
};

struct LatParams {
  int B, H, N, M, D;
  int tok_offset, n_global;     // this shard holds tokens [tok_offset, tok_offset + N) of n_global
  int q_per_batch;              // queries [G][M][D] with G = B*H (1) or H (0)
  int n_splits, tiles_per_split, rows_per_block;   // rows_per_block: 16 per warp, at most 128
  // scores in log2 units: t = smul * <qmul * q, k>, qmul * smul = scale * log2(e).
  // qmul = scale * log2(e), smul = 1: the query operand is pre-scaled (rounded
  // to tf32 with the scale); qmul = 1, smul = scale * log2(e): the product of
  // bf16-exact queries and keys is exact and the scale follows in fp32, as in
  // the forward's kernels (the gradient modes only)
  float qmul, smul;
  const int32_t* lengths;
  const float* q;               // fp32 queries [G][M][D]
  const float* zrow;            // decoder: Z [B*H][M][D]; encoder: dZ [B*H][M][D]
  const float* lrow;            // encoder: row log2-normaliser [B*H][M]
  const float* grow;            // encoder: gamma = <dZ, Z> [B*H][M]
  const uint16_t* k;            // bf16 [B*H][N][D]
  const uint16_t* v;            // bf16 [B*H][N][D] (forward, encoder)
  const uint16_t* dy;           // bf16 [B*H][N][D] (decoder)
  const float* ltok;            // decoder: per-token log2-normaliser [B*H][N]
  const float* dtok;            // decoder: delta = <dY, Y> [B*H][N]
  float* part_a;                // forward: [B*H][S][M][D+2]; decoder: dZ partials [B*H][S][M][D]
  float* part_b;                // decoder / encoder: dQ partials [B*H][S][M][D]
  uint32_t* err;
};

struct LatMergeParams {
  int BH, M, D, S;
  int R;                        // shards (ranks), partials rank-major
  size_t rank_stride;           // floats between two ranks' partials
  const float* part;            // [R][B*H][S][M][D+2]
  float* z;                     // [B*H][M][D]
  float* lse;                   // [B*H][M], log2 units
};

struct LatSumParams {
  int B, H, M, D, S;
  int fold_batch;               // 1: out [H][M][D] sums the batch; 0: out [B*H][M][D]
  float mult;
  const float* part0;           // [R][B*H][S][M][D] (rank-major)
  const float* part1;           // same shape or NULL
  const float* zref;            // [B*H][M][D] or NULL: gamma = <out, zref> per row
  float* gamma;                 // [B*H][M]
  float* out;                   // fp32: out = addend + mult * sum
  int R;                        // shards (ranks)
  size_t rank_stride;           // floats between two ranks' partials
  const float* addend;          // same shape as out, or NULL
};

// Modes of the token-parallel kernel (one CTA = kBwdTokBlock tokens of one
// head; a warp = one or two tiles of 16 token rows).
enum TokMode : int {
  kTokStats = 0,     // decoder recompute: per-token log2-normaliser and delta = <dY, Y>
  kTokFull = 1,      // dK (decoder + encoder parts) and dV
  kTokEncoder = 2,   // dK and dV of an encoder alone (the query synthesis)
};

struct TokParams {
  int B, H, N, M, D;
  int tok_offset, n_global;     // this shard holds tokens [tok_offset, tok_offset + N) of n_global
  int q_per_batch;
  float smul;                   // score multiplier: qpad holds (scale * log2(e) / smul) * q
  const int32_t* lengths;
  // padded tf32 images ([rows][D + 4], see PadParams)
  const float* qpad;            // scaled queries [G][M][D + 4]
  const float* zpad;            // Z [B*H][M][D + 4] (stats, full)
  const float* dzpad;           // dZ [B*H][M][D + 4] (full, encoder)
  const float* lm;              // encoder row log2-normaliser [B*H][M]
  const float* gam;             // gamma [B*H][M]
  const uint16_t *k, *v, *dy;   // bf16 [B*H][N][D]
  float* ltok;                  // [B*H][N]: written (stats), read (full)
  float* dtok;                  // [B*H][N]: written (stats), read (full)
  uint16_t *ghi, *glo;          // token-major gradient rows [B][N][g_ld] as bf16 high and low parts, or NULL
  int g_ld, g_col_k, g_col_v;   // row stride and column offsets of dK and dV (head h adds h*D)
  uint16_t* dk16;               // or bf16 [B*H][N][D] outputs
  uint16_t* dv16;
};

// Projection gradients on tcgen05 (proj_grad.cu).  G: the token-major
// gradient rows [R][4C] = [dK | dV | dK~ | dV~] (R = B*N) as two bf16
// planes, high and low parts; Wcat = [W_K | W_V | W~_K | W~_V], each [C][C].
// dX[r][c] = sum_j G[r][j] Wcat[c][j].
struct DxTcParams {
  int R, C;
  uint16_t* dx;                 // bf16 [R][C]
  uint32_t* err;
  unsigned long long timeout_ns;
};
// ghi, glo: [R][4C] bf16, 64 x 128 boxes, SW128; w[q]: W_q [C][C] bf16, 64 x C boxes, SW128.
struct DxTcMaps {
  CUtensorMap ghi, glo, w[4];
};
// Partials of the transposed weight gradient over splits of rows_per_split
// token rows: part[s][j][c] = sum_{r in split s} G[r][j] X[r][c].
struct DwTcParams {
  int R, C, n_splits, rows_per_split;
  float* part;                  // [n_splits][4C][C]
  uint32_t* err;
  unsigned long long timeout_ns;
};
// ghi, glo: [R][4C] bf16 and x: X [R][C] bf16, all 64 x 32 boxes, SW128.
struct DwTcMaps {
  CUtensorMap ghi, glo, x;
};

// dW_q[c][j] = sum_splits part[.][q*C + j][c] (+ part[.][(q+2)*C + j][c]
// when the synthesis weights are the encode weights).
struct DwReduceParams {
  int C, J, n_splits, shared;
  const float* part;
  float* dw[4];                 // [C][C] fp32 each (dWk, dWv, dWk_syn, dWv_syn); NULL = not written
};

// dst [rows][D + 4] = tf32(mul * src [rows][D]), the four pad columns zero.
struct PadParams {
  long rows;
  int D;
  float mul;
  const float* src;
  float* dst;
};

struct CvtParams {
  long n;
  const uint16_t* src;
  float* dst;
};

// Latent-parallel backward passes on tcgen05 (lat_tc.cu; D = 16, bf16
// queries, exact scores): the encoder's dQ partials, or the decoder's dQ and
// dZ partials, per (head, 128-latent block, token split).
constexpr int kLatTcEncoder = 0;
constexpr int kLatTcDecoder = 1;
struct LatTcParams {
  int B, H, N, M, D;
  int q_per_batch;              // queries [G][M][D] with G = B*H (1) or H (0)
  int n_lblocks, n_splits;
  int split_tokens;             // tokens per split (split s: [s*split_tokens, ...))
  int q_rows;                   // rows of one query box: min(M, kLatBlock)
  float c;                      // scale * log2(e), applied to the fp32 product
  const int32_t* lengths;
  const float* lrow;            // encoder: row log2-normaliser L_m [B*H][M]
  const float* grow;            // encoder: gamma_m [B*H][M]
  float* part_q;                // dQ partials [B*H][S][M][D]
  float* part_z;                // decoder: dZ partials [B*H][S][M][D]
  uint32_t* err;
  unsigned long long timeout_ns;
};
// Tensor maps: q (bf16 [G][M][D]); xa, xb (bf16 [B*H][M][D]: the high and low
// parts of dZ for the encoder, of Z for the decoder); k, u (bf16 [B*H][N][D]:
// K and V for the encoder, K and dY for the decoder); l, d (fp32 [B*H][N]:
// the decoder's L_n and delta_n).
struct LatTcMaps {
  CUtensorMap q, xa, xb, k, u, l, d;
};
cudaError_t launch_lat_tc(int mode, const LatTcMaps& m, const LatTcParams& p, cudaStream_t s);
size_t lat_tc_smem_bytes(int D);
int lat_tc_tile(int D);  // tokens per tile (the token maps' box rows)
// Token-parallel backward passes on tcgen05 (tok_tc.cu; D = 16, bf16
// queries, exact scores): dK and dV rows of 128-token tiles, the decoder and
// encoder parts (kTokTcFull) or the encoder part alone (kTokTcEncoder: the
// query synthesis).
constexpr int kTokTcFull = 0;
constexpr int kTokTcEncoder = 1;
struct TokTcParams {
  int B, H, N, M, D;
  int q_per_batch;              // queries [G][M][D] with G = B*H (1) or H (0)
  float c;                      // scale * log2(e), applied to the fp32 product
  const int32_t* lengths;
  const float* ltok;            // full: L_n [B*H][N]
  const float* dtok;            // full: delta_n [B*H][N]
  uint16_t *ghi, *glo;          // token-major gradient rows [B][N][g_ld] as bf16 high and low parts, or NULL
  int g_ld, g_col_k, g_col_v;   // row stride and column offsets of dK and dV (head h adds h*D)
  uint16_t *dk16, *dv16;        // or bf16 [B*H][N][D] outputs
  uint32_t* err;
  unsigned long long timeout_ns;
};
// Tensor maps: k, v, y (bf16 [B*H][N][D], 128-token boxes: K, V, dY); q (bf16
// [G][M][D]); zh, zl (Z's bf16 parts), dh, dl (dZ's, or dQ(X)'s for the
// synthesis) (bf16 [B*H][M][D]); lm, gm (fp32 [B*H][M]: L_m, gamma_m); all
// latent boxes tok_tc_chunk(mode) rows.
struct TokTcMaps {
  CUtensorMap k, v, y, q, zh, zl, dh, dl, lm, gm;
};
cudaError_t launch_tok_tc(int mode, const TokTcMaps& m, const TokTcParams& p, cudaStream_t s);
size_t tok_tc_smem_bytes(int mode, int D);
int tok_tc_chunk(int mode, int D);  // latents per ring stage (the latent tensor maps' box rows)

// hi[i] = bf16(x[i]), lo[i] = bf16(x[i] - hi[i]) for i < n (n even)
struct SplitHiLoParams {
  long n;
  const float* x;
  uint16_t *hi, *lo;
};
cudaError_t launch_split_hilo(const SplitHiLoParams& p, cudaStream_t s);

// delta_n = <dY_n, Y_n> per token from a training forward's fp32 Y (0 for
// padding tokens).
struct DeltaParams {
  int B, H, N, D;
  int tok_offset, n_global;
  const int32_t* lengths;
  const float* y32;             // [B*H][N][D]
  const uint16_t* dy;           // bf16 [B*H][N][D]
  float* dtok;                  // [B*H][N]
};
cudaError_t launch_delta(const DeltaParams& p, cudaStream_t s);

// The mark a training forward leaves in its workspace; a training backward
// that does not find it sets FLARE_DEV_NO_STATE in the error word.
struct MarkParams {
  const uint32_t* mark;         // must hold kTrainStateTag
  uint32_t* err;
};
constexpr int kTrainStateByte = 0xA5;               // written with a byte memset
constexpr uint32_t kTrainStateTag = 0xA5A5A5A5u;    // kTrainStateByte in all four bytes

cudaError_t launch_lat(int mode, const LatParams& p, cudaStream_t s);
cudaError_t launch_check_mark(const MarkParams& p, cudaStream_t s);
cudaError_t launch_lat_merge(const LatMergeParams& p, cudaStream_t s);
cudaError_t launch_lat_sum(const LatSumParams& p, cudaStream_t s);
cudaError_t launch_tok(int mode, const TokParams& p, cudaStream_t s);
cudaError_t launch_dx_tc(const DxTcMaps& m, const DxTcParams& p, cudaStream_t s);
cudaError_t launch_dw_tc(const DwTcMaps& m, const DwTcParams& p, cudaStream_t s);
cudaError_t launch_dw_tc_reduce(const DwReduceParams& p, cudaStream_t s);
cudaError_t launch_pad(const PadParams& p, cudaStream_t s);
cudaError_t launch_cvt(const CvtParams& p, cudaStream_t s);

}  // namespace flare
