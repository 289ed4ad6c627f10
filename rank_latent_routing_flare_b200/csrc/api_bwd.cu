// Host entry points of the C ABI for the backward (gradients): argument
// validation, the backward's workspace plan and the launch sequences of
// flare_mixer_bwd, flarepp_mixer_bwd and the context-parallel phases of the
// FLARE++ backward (flarepp_cp_bwd_phase).  The kernels are in backward.cu.
#include <algorithm>
#include <cmath>

#include "bwd_internal.h"
#include "flare.h"
#include "flare_internal.h"
#include "host_internal.h"

namespace flare {

BwdPlan make_bwd_plan(bool pp, long B, long H, long N, long M, long D, long C) {
  BwdPlan bp;
  bp.fwd = make_plan(pp ? FLARE_VARIANT_FLAREPP : FLARE_VARIANT_FLARE, B, H, N, M, D);
  const long BH = B * H;
  // latent-parallel passes: 32, 64, 96 or 128 latent rows per CTA, so that
  // both a warp per 16 rows and a warp per 32 rows give whole warps
  bp.rpb = static_cast<int>(std::min(128L, cdiv(M, 32) * 32));
  bp.LB = static_cast<int>(cdiv(M, bp.rpb));
  // token splits: whole waves of CTAs (about 128 registers per thread, so
  // 256 / rows_per_block CTAs per SM), by the encoder's cost model
  const long ntiles = cdiv(N, kBwdTokTile);
  bp.S = choose_splits(BH * bp.LB, ntiles, static_cast<long>(kNumSM) * std::max(1, 256 / bp.rpb), 8);
  bp.tps = static_cast<int>(cdiv(ntiles, bp.S));
  bp.S = static_cast<int>(cdiv(ntiles, bp.tps));
  bp.dw_splits = static_cast<int>(cdiv(B * N, kBwdDwRows));
  size_t off = bp.fwd.total;
  auto take = [&off](size_t bytes) {
    const size_t o = off;
    off += align256(bytes);
    return o;
  };
  const size_t lat = static_cast<size_t>(BH * M * D) * 4, row = static_cast<size_t>(BH * M) * 4;
  const size_t tokv = static_cast<size_t>(BH * N) * 4;
  const size_t part = static_cast<size_t>(BH) * bp.S * M * D * 4;
  bp.off_q32 = take(static_cast<size_t>(H * M * D) * 4);
  if (pp) {
    bp.off_qx32 = take(lat);
    bp.off_lsyn = take(row);
    bp.off_dqx32 = take(lat);
    bp.off_gsyn = take(row);
  }
  bp.off_z32 = take(lat);
  bp.off_lenc = take(row);
  bp.off_ltok = take(tokv);
  bp.off_dtok = take(tokv);
  bp.off_dz32 = take(lat);
  bp.off_gam = take(row);
  bp.off_fpart = take(static_cast<size_t>(BH) * bp.S * M * (D + 2) * 4);
  bp.off_pa = take(2 * part);  // [dZ partials | dQ partials] of the decoder backward
  bp.off_pc = take(part);
  // padded tf32 images ([rows][D + 4]) read by the token-parallel pass
  const size_t padded = static_cast<size_t>(BH * M * (D + 4)) * 4;
  bp.off_qpad = take(padded);
  bp.off_zpad = take(padded);
  bp.off_dzpad = take(padded);
  if (pp) {
    bp.off_q0pad = take(static_cast<size_t>(H * M * (D + 4)) * 4);
    bp.off_dqxpad = take(padded);
  }
  // FLARE++: the decoder's part of dQ(X) [B*H][M][D]; FLARE: the decoder's
  // part of dQ, summed over the batch [H][M][D]
  bp.off_dqxdec = take(lat);
  if (pp) {
    // the gradient rows [B*N][4C] = [dK | dV | dK~ | dV~] as two bf16 planes
    // (high and low parts), read by the projection gradients
    bp.off_grows = take(static_cast<size_t>(B * N) * 4 * C * 4);
    bp.off_dwpart = take(static_cast<size_t>(bp.dw_splits) * C * 4 * C * 4);
  }
  // the high and low bf16 parts of dZ (then of dQ(X)) and of Z for the
  // tcgen05 passes of the training backward
  bp.off_xhi16 = take(static_cast<size_t>(BH * M * D) * 2);
  bp.off_xlo16 = take(static_cast<size_t>(BH * M * D) * 2);
  bp.off_zhi16 = take(static_cast<size_t>(BH * M * D) * 2);
  bp.off_zlo16 = take(static_cast<size_t>(BH * M * D) * 2);
  // the training pair at D = 16: the forward's fp16 copy of Z and its fp32 Y
  // (FLARE++: in the gradient rows' space, which the backward fills only
  // after it has taken delta_n from Y)
  if (D == 16) {
    bp.off_zf16 = take(static_cast<size_t>(BH * M * D) * 2);
    bp.off_y32 = pp ? bp.off_grows : take(static_cast<size_t>(BH * N * D) * 4);
  }
  bp.total = off;
  return bp;
}

}  // namespace flare

// ---------------------------------------------------------------------------
// Backward (gradients)
// ---------------------------------------------------------------------------

namespace flare {
namespace {

constexpr float kLog2e = 1.4426950408889634f;

// Where the token-parallel pass writes dK and dV: token-major fp32 rows of
// the projection-gradient matrix, or bf16 [B][H][N][D] outputs.
struct TokOut {
  float* g32;
  int g_ld, col_k, col_v;
  uint16_t *dk16, *dv16;
};

// This GPU's token shard: tokens [tok_offset, tok_offset + N) of sequences
// of n_global tokens, one of R shards (R = 1: the whole sequence).
struct Shard {
  int tok_offset, n_global, R;
};

LatParams lat_params(const BwdPlan& bp, uint8_t* ws, const float* q, int q_per_batch, const void* k, int B, int H,
                     int N, int M, int D, const int32_t* lengths, float sc, const Shard& sh) {
  LatParams lp{};
  lp.B = B; lp.H = H; lp.N = N; lp.M = M; lp.D = D;
  lp.tok_offset = sh.tok_offset; lp.n_global = sh.n_global;
  lp.q_per_batch = q_per_batch;
  lp.n_splits = bp.S; lp.tiles_per_split = bp.tps; lp.rows_per_block = bp.rpb;
  lp.qmul = sc * kLog2e;
  lp.smul = 1.f;
  lp.lengths = lengths;
  lp.q = q;
  lp.k = static_cast<const uint16_t*>(k);
  lp.err = reinterpret_cast<uint32_t*>(ws + bp.fwd.off_err);
  return lp;
}

TokParams tok_params(int B, int H, int N, int M, int D, int q_per_batch, const int32_t* lengths, float sc,
                     const Shard& sh) {
  TokParams tp{};
  tp.B = B; tp.H = H; tp.N = N; tp.M = M; tp.D = D;
  tp.tok_offset = sh.tok_offset; tp.n_global = sh.n_global;
  tp.q_per_batch = q_per_batch;
  tp.smul = 1.f;
  tp.lengths = lengths;
  return tp;
}

// out = addend + mult * (sum over R shards and S splits of part0 (+ part1)),
// gamma = <out, zref> per row when zref is given.
flare_status lat_sum(int B, int H, int M, int D, int S, int fold_batch, float mult, const float* part0,
                     const float* part1, int R, size_t rank_stride, const float* addend, const float* zref,
                     float* gamma, float* out, cudaStream_t s) {
  LatSumParams p{};
  p.B = B; p.H = H; p.M = M; p.D = D; p.S = S;
  p.fold_batch = fold_batch; p.mult = mult;
  p.part0 = part0; p.part1 = part1; p.zref = zref; p.gamma = gamma; p.out = out;
  p.R = R; p.rank_stride = rank_stride; p.addend = addend;
  return launch_lat_sum(p, s) == cudaSuccess ? FLARE_OK : FLARE_ERR_LAUNCH;
}

// Merge of the recompute partials of R shards: Z (or Q(X)) and L_m.
flare_status lat_merge(const float* part, int R, size_t rank_stride, int BH, int M, int D, int S, float* z,
                       float* lse, cudaStream_t s) {
  LatMergeParams mp{};
  mp.BH = BH; mp.M = M; mp.D = D; mp.S = S;
  mp.R = R; mp.rank_stride = rank_stride;
  mp.part = part; mp.z = z; mp.lse = lse;
  return launch_lat_merge(mp, s) == cudaSuccess ? FLARE_OK : FLARE_ERR_LAUNCH;
}

// Exact scores for the gradient modes (see LatParams): the query operand
// unscaled, the scale applied to the fp32 product.  The training backward
// uses them so that its scores match the forward's, whose normalisers it
// reuses.
void exact_scores(LatParams& lp, float sc) {
  lp.qmul = 1.f;
  lp.smul = sc * kLog2e;
}

#ifndef FLARE_LAT_TC
#define FLARE_LAT_TC 1
#endif
// The training backward's latent-parallel passes at D = 16 run on tcgen05
// (lat_tc.cu) unless built with FLARE_LAT_TC=0 (the tf32 passes, kept for D = 32
// and the self-contained backward).
bool use_lat_tc(bool exact, int D) { return FLARE_LAT_TC && exact && (D == 16 || D == 32); }

// One tcgen05 latent-parallel pass: q16 bf16 queries ([G][M][D]), xa16 / xb16
// the high and low parts of dZ (encoder) or Z (decoder), k16 / u16 the token
// rows (K and V, or K and dY), and for the decoder L_n, delta_n; partials as
// the tf32 passes write them ([B*H][S][M][D], S = bp.S splits of bp.tps
// 64-token tiles).
flare_status lat_tc(int mode, const BwdPlan& bp, uint8_t* ws, const void* q16, int q_per_batch, const void* xa16,
                    const void* xb16, const void* k16, const void* u16, const float* ltok, const float* dtok,
                    const float* lrow, const float* grow, float* part_q, float* part_z, int B, int H, int N, int M,
                    int D, const int32_t* lengths, float sc, cudaStream_t s) {
  const long BH = static_cast<long>(B) * H;
  const long G = q_per_batch ? BH : H;
  const int qrows = std::min(M, kLatBlock), T = lat_tc_tile(D);
  LatTcMaps mp;
  if (!map3d(&mp.q, q16, D, M, G, D, qrows, row_swizzle(D)) || !map3d(&mp.xa, xa16, D, M, BH, D, qrows, row_swizzle(D)) ||
      !map3d(&mp.xb, xb16, D, M, BH, D, qrows, row_swizzle(D)) || !map3d(&mp.k, k16, D, N, BH, D, T, row_swizzle(D)) ||
      !map3d(&mp.u, u16, D, N, BH, D, T, row_swizzle(D)))
    return FLARE_ERR_LAUNCH;
  if (mode == kLatTcDecoder && (!map2d_f32(&mp.l, ltok, N, BH, T, 1) || !map2d_f32(&mp.d, dtok, N, BH, T, 1)))
    return FLARE_ERR_LAUNCH;
  LatTcParams p{};
  p.B = B; p.H = H; p.N = N; p.M = M; p.D = D;
  p.q_per_batch = q_per_batch;
  p.n_lblocks = static_cast<int>(cdiv(M, kLatBlock));
  p.n_splits = bp.S;
  p.split_tokens = bp.tps * kBwdTokTile;
  p.q_rows = qrows;
  p.c = sc * kLog2e;
  p.lengths = lengths;
  p.lrow = lrow; p.grow = grow;
  p.part_q = part_q; p.part_z = part_z;
  p.err = reinterpret_cast<uint32_t*>(ws + bp.fwd.off_err);
  p.timeout_ns = wait_timeout_ns();
  return launch_lat_tc(mode, mp, p, s) == cudaSuccess ? FLARE_OK : FLARE_ERR_LAUNCH;
}

// x (fp32 [rows][D]) into the high and low bf16 parts kept for the tcgen05
// passes (dZ, then dQ(X): the x buffers; Z: the z buffers).
flare_status split_hilo(const BwdPlan& bp, uint8_t* ws, const float* x, long n, cudaStream_t s, bool z = false) {
  const SplitHiLoParams sp{n, x, reinterpret_cast<uint16_t*>(ws + (z ? bp.off_zhi16 : bp.off_xhi16)),
                           reinterpret_cast<uint16_t*>(ws + (z ? bp.off_zlo16 : bp.off_xlo16))};
  return launch_split_hilo(sp, s) == cudaSuccess ? FLARE_OK : FLARE_ERR_LAUNCH;
}

// One tcgen05 token-parallel pass (see TokTcParams): dK, dV rows into ghi /
// glo (token-major rows as bf16 high and low parts) or into bf16 dk16 / dv16.  Full: z parts from the
// z buffers, L_n and delta_n; both modes: the dZ (or dQ(X)) parts from the x
// buffers, L_m and gamma_m.
flare_status tok_tc(int mode, const BwdPlan& bp, uint8_t* ws, const void* k16, const void* v16, const void* dy16,
                    const void* q16, int q_per_batch, const float* ltok, const float* dtok, const float* lm,
                    const float* gm, uint16_t* ghi, uint16_t* glo, int g_ld, int g_col_k, int g_col_v, uint16_t* dk16, uint16_t* dv16,
                    int B, int H, int N, int M, int D, const int32_t* lengths, float sc, cudaStream_t s) {
  const long BH = static_cast<long>(B) * H;
  const long G = q_per_batch ? BH : H;
  const CUtensorMapSwizzle sw = row_swizzle(D);
  TokTcMaps mp;
  const bool full = mode == kTokTcFull;
  const uint32_t ch = static_cast<uint32_t>(tok_tc_chunk(mode, D));
  if (!map3d(&mp.k, k16, D, N, BH, D, kBwdTokBlock, sw) || !map3d(&mp.v, v16, D, N, BH, D, kBwdTokBlock, sw) ||
      !map3d(&mp.y, full ? dy16 : k16, D, N, BH, D, kBwdTokBlock, sw) || !map3d(&mp.q, q16, D, M, G, D, ch, sw) ||
      !map3d(&mp.zh, ws + bp.off_zhi16, D, M, BH, D, ch, sw) || !map3d(&mp.zl, ws + bp.off_zlo16, D, M, BH, D, ch, sw) ||
      !map3d(&mp.dh, ws + bp.off_xhi16, D, M, BH, D, ch, sw) || !map3d(&mp.dl, ws + bp.off_xlo16, D, M, BH, D, ch, sw) ||
      !map2d_f32(&mp.lm, lm, M, BH, ch, 1) || !map2d_f32(&mp.gm, gm, M, BH, ch, 1))
    return FLARE_ERR_LAUNCH;
  TokTcParams p{};
  p.B = B; p.H = H; p.N = N; p.M = M; p.D = D;
  p.q_per_batch = q_per_batch;
  p.c = sc * kLog2e;
  p.lengths = lengths;
  p.ltok = ltok; p.dtok = dtok;
  p.ghi = ghi; p.glo = glo; p.g_ld = g_ld; p.g_col_k = g_col_k; p.g_col_v = g_col_v;
  p.dk16 = dk16; p.dv16 = dv16;
  p.err = reinterpret_cast<uint32_t*>(ws + bp.fwd.off_err);
  p.timeout_ns = wait_timeout_ns();
  return launch_tok_tc(mode, mp, p, s) == cudaSuccess ? FLARE_OK : FLARE_ERR_LAUNCH;
}

flare_status pad(const float* src, float* dst, long rows, int D, float mul, cudaStream_t s) {
  const PadParams pp{rows, D, mul, src, dst};
  return launch_pad(pp, s) == cudaSuccess ? FLARE_OK : FLARE_ERR_LAUNCH;
}

// fp32 elements of one split-partials buffer [B*H][S][M][D] (+2 per row for
// the recompute partials).
size_t part_floats(const BwdPlan& bp, int B, int H, int M, int D, bool recompute) {
  return static_cast<size_t>(B) * H * bp.S * M * (D + (recompute ? 2 : 0));
}

// ---------------------------------------------------------------------------
// FLARE (eq. 5-6) backward in four phases, like the FLARE++ one below: between
// two phases every shard's exchange buffer is all-gathered in rank order and
// merged in ascending (rank, split) order, so every rank holds bitwise the
// same Z, dZ and dQ.  On one GPU the phases run back to back with the
// exchanges in the workspace.
//   0: encoder recompute partials of the shard's tokens            -> E0
//   1: merge E0 -> Z, L_m; decoder stats; decoder backward         -> E1 = [dZ | dQ_dec partials]
//   2: dZ, gamma, scale * dQ_dec (summed over the batch); dK, dV of
//      the shard's tokens (bf16 outputs); encoder dQ partials      -> E2
//   3: dQ = scale * dQ_enc + the decoder part, summed over the batch
// ---------------------------------------------------------------------------
constexpr int kFlPhases = 4;

struct FlArgs {
  const flare_bf16 *K, *V, *Q, *dY;
  flare_bf16 *dK, *dV;
  float* dQ;
  int B, H, N, M, D;
  const int32_t* lengths;
  float sc;
  Shard sh;
  bool exact = false;  // exact scores (the training backward), see exact_scores
};

size_t fl_exchange_floats(const BwdPlan& bp, int phase, int B, int H, int M, int D) {
  switch (phase) {
    case 0: return part_floats(bp, B, H, M, D, true);
    case 1: return 2 * part_floats(bp, B, H, M, D, false);
    case 2: return part_floats(bp, B, H, M, D, false);
    default: return 0;
  }
}

flare_status fl_phase(int phase, const BwdPlan& bp, uint8_t* ws, const FlArgs& a, const float* gathered, float* exch,
                      cudaStream_t s) {
  const int B = a.B, H = a.H, N = a.N, M = a.M, D = a.D;
  const long BH = static_cast<long>(B) * H;
  const float sc = a.sc, c = sc * kLog2e;
  const int R = a.sh.R;
  float* q32 = reinterpret_cast<float*>(ws + bp.off_q32);
  float* z32 = reinterpret_cast<float*>(ws + bp.off_z32);
  float* lenc = reinterpret_cast<float*>(ws + bp.off_lenc);
  float* ltok = reinterpret_cast<float*>(ws + bp.off_ltok);
  float* dtok = reinterpret_cast<float*>(ws + bp.off_dtok);
  float* dz32 = reinterpret_cast<float*>(ws + bp.off_dz32);
  float* gam = reinterpret_cast<float*>(ws + bp.off_gam);
  float* dqdec = reinterpret_cast<float*>(ws + bp.off_dqxdec);
  float* qpad = reinterpret_cast<float*>(ws + bp.off_qpad);
  float* zpad = reinterpret_cast<float*>(ws + bp.off_zpad);
  float* dzpad = reinterpret_cast<float*>(ws + bp.off_dzpad);
  const uint16_t* k = reinterpret_cast<const uint16_t*>(a.K);
  const uint16_t* v = reinterpret_cast<const uint16_t*>(a.V);
  const uint16_t* dy = reinterpret_cast<const uint16_t*>(a.dY);
  const size_t P = part_floats(bp, B, H, M, D, false);
  const size_t stride = fl_exchange_floats(bp, phase - 1, B, H, M, D);  // of the gathered buffers
  flare_status st = FLARE_OK;
  switch (phase) {
    case 0: {
      if (cudaMemsetAsync(ws + bp.fwd.off_err, 0, kErrClearBytes, s) != cudaSuccess) return FLARE_ERR_LAUNCH;
      const CvtParams cv{static_cast<long>(H) * M * D, reinterpret_cast<const uint16_t*>(a.Q), q32};
      if (launch_cvt(cv, s) != cudaSuccess) return FLARE_ERR_LAUNCH;
      // eq. 5 recomputed: the encoder partials of this shard
      LatParams lf = lat_params(bp, ws, q32, 0, k, B, H, N, M, D, a.lengths, sc, a.sh);
      lf.v = v;
      lf.part_a = exch;
      return launch_lat(kLatForward, lf, s) == cudaSuccess ? FLARE_OK : FLARE_ERR_LAUNCH;
    }
    case 1: {
      if ((st = lat_merge(gathered, R, stride, static_cast<int>(BH), M, D, bp.S, z32, lenc, s)) != FLARE_OK ||
          (st = pad(q32, qpad, static_cast<long>(H) * M, D, c, s)) != FLARE_OK ||
          (st = pad(z32, zpad, BH * M, D, 1.f, s)) != FLARE_OK)
        return st;
      // eq. 6: the decoder's per-token normalisers and delta_n of this shard
      TokParams tp = tok_params(B, H, N, M, D, 0, a.lengths, sc, a.sh);
      tp.qpad = qpad; tp.zpad = zpad;
      tp.k = k; tp.v = v; tp.dy = dy;
      tp.ltok = ltok; tp.dtok = dtok;
      if (launch_tok(kTokStats, tp, s) != cudaSuccess) return FLARE_ERR_LAUNCH;
      // decoder backward, reductions over this shard's tokens: dZ and dQ partials
      LatParams ld = lat_params(bp, ws, q32, 0, k, B, H, N, M, D, a.lengths, sc, a.sh);
      ld.zrow = z32; ld.dy = dy; ld.ltok = ltok; ld.dtok = dtok;
      ld.part_a = exch; ld.part_b = exch + P;
      return launch_lat(kLatDecoder, ld, s) == cudaSuccess ? FLARE_OK : FLARE_ERR_LAUNCH;
    }
    case 2: {
      // dZ and gamma; the decoder's part of dQ, scaled and summed over the batch
      if ((st = lat_sum(B, H, M, D, bp.S, 0, 1.f, gathered, nullptr, R, stride, nullptr, z32, gam, dz32, s)) !=
              FLARE_OK ||
          (st = lat_sum(B, H, M, D, bp.S, 1, sc, gathered + P, nullptr, R, stride, nullptr, nullptr, nullptr, dqdec,
                        s)) != FLARE_OK ||
          (st = pad(dz32, dzpad, BH * M, D, 1.f, s)) != FLARE_OK)
        return st;
      // dK (both parts) and dV of this shard's tokens
      TokParams tp = tok_params(B, H, N, M, D, 0, a.lengths, sc, a.sh);
      tp.qpad = qpad; tp.zpad = zpad; tp.dzpad = dzpad; tp.lm = lenc; tp.gam = gam;
      tp.k = k; tp.v = v; tp.dy = dy;
      tp.ltok = ltok; tp.dtok = dtok;
      tp.dk16 = reinterpret_cast<uint16_t*>(a.dK);
      tp.dv16 = reinterpret_cast<uint16_t*>(a.dV);
      if (use_lat_tc(a.exact, D)) {  // both passes on tcgen05, from the parts of dZ (and Z)
        if ((st = split_hilo(bp, ws, dz32, BH * M * D, s)) != FLARE_OK ||
            (st = tok_tc(kTokTcFull, bp, ws, k, v, dy, a.Q, 0, ltok, dtok, lenc, gam, nullptr, nullptr, 0, 0, 0,
                         reinterpret_cast<uint16_t*>(a.dK), reinterpret_cast<uint16_t*>(a.dV), B, H, N, M, D,
                         a.lengths, sc, s)) != FLARE_OK)
          return st;
        return lat_tc(kLatTcEncoder, bp, ws, a.Q, 0, ws + bp.off_xhi16, ws + bp.off_xlo16, k, v, nullptr, nullptr,
                      lenc, gam, exch, nullptr, B, H, N, M, D, a.lengths, sc, s);
      }
      if (a.exact) tp.smul = c;
      if (launch_tok(kTokFull, tp, s) != cudaSuccess) return FLARE_ERR_LAUNCH;
      // encoder backward: its dQ partials
      LatParams le = lat_params(bp, ws, q32, 0, k, B, H, N, M, D, a.lengths, sc, a.sh);
      le.zrow = dz32; le.lrow = lenc; le.grow = gam; le.v = v;
      if (a.exact) exact_scores(le, sc);
      le.part_b = exch;
      return launch_lat(kLatEncoder, le, s) == cudaSuccess ? FLARE_OK : FLARE_ERR_LAUNCH;
    }
    case 3:
      // dQ = scale * (decoder + encoder parts), summed over the batch and the shards
      return lat_sum(B, H, M, D, bp.S, 1, sc, gathered, nullptr, R, stride, dqdec, nullptr, nullptr, a.dQ, s);
    default:
      return FLARE_ERR_SHAPE;
  }
}

// ---------------------------------------------------------------------------
// FLARE++ (eq. 7-11) backward in seven phases.  Between two phases every
// shard's exchange buffer is all-gathered in rank order; the next phase reads
// the gathered buffers (R shards, `stride` floats apart) and merges them in
// ascending (rank, split) order, so every rank holds bitwise the same Q(X),
// Z, dZ, dQ(X), dQ0 and dW.  On one GPU the phases run back to back with the
// exchanges in the workspace.  The workspace carries the shard's state
// (projections, Q(X), Z, normalisers, gradient rows) from phase to phase.
//   0: projections; synthesis recompute partials                 -> E0
//   1: merge E0 -> Q(X), L~_m; encode recompute partials         -> E1
//   2: merge E1 -> Z, L_m; decoder stats; decoder backward       -> E2 = [dZ | dQ_dec partials]
//   3: dZ, gamma, scale * dQ_dec; dK, dV rows; encoder dQ        -> E3
//   4: dQ(X), gamma~; dK~, dV~ rows; synthesis dQ0 partials      -> E4
//   5: dQ0; dX (local rows); dW partials of the local rows       -> E5
//   6: dW
// ---------------------------------------------------------------------------
constexpr int kPpPhases = 7;

struct PpArgs {
  const flare_bf16 *X, *Wk, *Wv, *Wk_syn, *Wv_syn, *Q0, *dY;
  flare_bf16* dX;
  float *dWk, *dWv, *dWk_syn, *dWv_syn, *dQ0;
  int B, N, C, H, M, D;
  const int32_t* lengths;
  float sc;
  Shard sh;
  bool exact = false;  // exact scores (the training backward), see exact_scores
};

size_t pp_exchange_floats(const BwdPlan& bp, int phase, int B, int H, int M, int D, int C) {
  switch (phase) {
    case 0:
    case 1: return part_floats(bp, B, H, M, D, true);
    case 2: return 2 * part_floats(bp, B, H, M, D, false);
    case 3:
    case 4: return part_floats(bp, B, H, M, D, false);
    case 5: return static_cast<size_t>(bp.dw_splits) * C * 4 * C;
    default: return 0;
  }
}

flare_status pp_phase(int phase, const BwdPlan& bp, uint8_t* ws, const PpArgs& a, const float* gathered,
                      float* exch, cudaStream_t s) {
  const int B = a.B, N = a.N, C = a.C, H = a.H, M = a.M, D = a.D;
  const long BH = static_cast<long>(B) * H;
  const float sc = a.sc, c = sc * kLog2e;
  const int R = a.sh.R;
  const bool shared = a.Wk_syn == a.Wk && a.Wv_syn == a.Wv;
  uint16_t* kk = reinterpret_cast<uint16_t*>(ws + bp.fwd.off_kp);
  uint16_t* vv = reinterpret_cast<uint16_t*>(ws + bp.fwd.off_vp);
  uint16_t* kt = shared ? kk : reinterpret_cast<uint16_t*>(ws + bp.fwd.off_kt);
  uint16_t* vt = shared ? vv : reinterpret_cast<uint16_t*>(ws + bp.fwd.off_vt);
  float* q32 = reinterpret_cast<float*>(ws + bp.off_q32);
  float* qx32 = reinterpret_cast<float*>(ws + bp.off_qx32);
  float* lsyn = reinterpret_cast<float*>(ws + bp.off_lsyn);
  float* z32 = reinterpret_cast<float*>(ws + bp.off_z32);
  float* lenc = reinterpret_cast<float*>(ws + bp.off_lenc);
  float* ltok = reinterpret_cast<float*>(ws + bp.off_ltok);
  float* dtok = reinterpret_cast<float*>(ws + bp.off_dtok);
  float* dz32 = reinterpret_cast<float*>(ws + bp.off_dz32);
  float* gam = reinterpret_cast<float*>(ws + bp.off_gam);
  float* dqx32 = reinterpret_cast<float*>(ws + bp.off_dqx32);
  float* dqxdec = reinterpret_cast<float*>(ws + bp.off_dqxdec);
  float* gsyn = reinterpret_cast<float*>(ws + bp.off_gsyn);
  float* qpad = reinterpret_cast<float*>(ws + bp.off_qpad);
  float* zpad = reinterpret_cast<float*>(ws + bp.off_zpad);
  float* dzpad = reinterpret_cast<float*>(ws + bp.off_dzpad);
  float* q0pad = reinterpret_cast<float*>(ws + bp.off_q0pad);
  float* dqxpad = reinterpret_cast<float*>(ws + bp.off_dqxpad);
  // the gradient rows [B*N][4C] as bf16 high and low planes
  uint16_t* ghi = reinterpret_cast<uint16_t*>(ws + bp.off_grows);
  uint16_t* glo = ghi + static_cast<size_t>(B) * N * 4 * C;
  const size_t P = part_floats(bp, B, H, M, D, false);
  const size_t stride = pp_exchange_floats(bp, phase - 1, B, H, M, D, C);  // of the gathered buffers
  flare_status st = FLARE_OK;
  switch (phase) {
    case 0: {
      if (cudaMemsetAsync(ws + bp.fwd.off_err, 0, kErrClearBytes, s) != cudaSuccess) return FLARE_ERR_LAUNCH;
      // eq. 7 and 9: the projections, recomputed (tcgen05, as in the forward)
      Projected pr;
      if ((st = flarepp_project(bp.fwd, a.X, a.Wk, a.Wv, a.Wk_syn, a.Wv_syn, B, N, C, H, D, ws, s, nullptr, &pr)) !=
          FLARE_OK)
        return st;
      const CvtParams cv{static_cast<long>(H) * M * D, reinterpret_cast<const uint16_t*>(a.Q0), q32};
      if (launch_cvt(cv, s) != cudaSuccess) return FLARE_ERR_LAUNCH;
      // eq. 8 recomputed: the synthesis partials of this shard
      LatParams lf = lat_params(bp, ws, q32, 0, kt, B, H, N, M, D, a.lengths, sc, a.sh);
      lf.v = vt;
      lf.part_a = exch;
      return launch_lat(kLatForward, lf, s) == cudaSuccess ? FLARE_OK : FLARE_ERR_LAUNCH;
    }
    case 1: {
      if ((st = lat_merge(gathered, R, stride, static_cast<int>(BH), M, D, bp.S, qx32, lsyn, s)) != FLARE_OK)
        return st;
      // eq. 10 recomputed: the encode partials of this shard
      LatParams lf = lat_params(bp, ws, qx32, 1, kk, B, H, N, M, D, a.lengths, sc, a.sh);
      lf.v = vv;
      lf.part_a = exch;
      return launch_lat(kLatForward, lf, s) == cudaSuccess ? FLARE_OK : FLARE_ERR_LAUNCH;
    }
    case 2: {
      if ((st = lat_merge(gathered, R, stride, static_cast<int>(BH), M, D, bp.S, z32, lenc, s)) != FLARE_OK ||
          (st = pad(qx32, qpad, BH * M, D, c, s)) != FLARE_OK || (st = pad(z32, zpad, BH * M, D, 1.f, s)) != FLARE_OK)
        return st;
      // eq. 11: the decoder's per-token normalisers and delta_n
      TokParams tp = tok_params(B, H, N, M, D, 1, a.lengths, sc, a.sh);
      tp.qpad = qpad; tp.zpad = zpad;
      tp.k = kk; tp.dy = reinterpret_cast<const uint16_t*>(a.dY);
      tp.ltok = ltok; tp.dtok = dtok;
      if (launch_tok(kTokStats, tp, s) != cudaSuccess) return FLARE_ERR_LAUNCH;
      // decoder backward, reductions over this shard's tokens: dZ and dQ(X) partials
      LatParams ld = lat_params(bp, ws, qx32, 1, kk, B, H, N, M, D, a.lengths, sc, a.sh);
      ld.zrow = z32; ld.dy = tp.dy; ld.ltok = ltok; ld.dtok = dtok;
      ld.part_a = exch; ld.part_b = exch + P;
      return launch_lat(kLatDecoder, ld, s) == cudaSuccess ? FLARE_OK : FLARE_ERR_LAUNCH;
    }
    case 3: {
      // dZ and gamma; the decoder's part of dQ(X)
      if ((st = lat_sum(B, H, M, D, bp.S, 0, 1.f, gathered, nullptr, R, stride, nullptr, z32, gam, dz32, s)) !=
              FLARE_OK ||
          (st = lat_sum(B, H, M, D, bp.S, 0, sc, gathered + P, nullptr, R, stride, nullptr, nullptr, nullptr,
                        dqxdec, s)) != FLARE_OK ||
          (st = pad(dz32, dzpad, BH * M, D, 1.f, s)) != FLARE_OK)
        return st;
      // dK (both parts) and dV of this shard's tokens, into the gradient rows
      TokParams tp = tok_params(B, H, N, M, D, 1, a.lengths, sc, a.sh);
      tp.qpad = qpad; tp.zpad = zpad; tp.dzpad = dzpad; tp.lm = lenc; tp.gam = gam;
      tp.k = kk; tp.v = vv; tp.dy = reinterpret_cast<const uint16_t*>(a.dY);
      tp.ltok = ltok; tp.dtok = dtok;
      tp.ghi = ghi; tp.glo = glo; tp.g_ld = 4 * C; tp.g_col_k = 0; tp.g_col_v = C;
      if (use_lat_tc(a.exact, D)) {  // both passes on tcgen05 (the forward's bf16 Q(X), the parts of dZ and Z)
        if ((st = split_hilo(bp, ws, dz32, BH * M * D, s)) != FLARE_OK ||
            (st = tok_tc(kTokTcFull, bp, ws, kk, vv, a.dY, ws + bp.fwd.off_qx16, 1, ltok, dtok, lenc, gam, ghi, glo,
                         4 * C, 0, C, nullptr, nullptr, B, H, N, M, D, a.lengths, sc, s)) != FLARE_OK)
          return st;
        return lat_tc(kLatTcEncoder, bp, ws, ws + bp.fwd.off_qx16, 1, ws + bp.off_xhi16, ws + bp.off_xlo16, kk, vv,
                      nullptr, nullptr, lenc, gam, exch, nullptr, B, H, N, M, D, a.lengths, sc, s);
      }
      if (a.exact) tp.smul = c;
      if (launch_tok(kTokFull, tp, s) != cudaSuccess) return FLARE_ERR_LAUNCH;
      // encoder backward: its dQ(X) partials
      LatParams le = lat_params(bp, ws, qx32, 1, kk, B, H, N, M, D, a.lengths, sc, a.sh);
      le.zrow = dz32; le.lrow = lenc; le.grow = gam; le.v = vv;
      if (a.exact) exact_scores(le, sc);
      le.part_b = exch;
      return launch_lat(kLatEncoder, le, s) == cudaSuccess ? FLARE_OK : FLARE_ERR_LAUNCH;
    }
    case 4: {
      // dQ(X) = scale * (decoder + encoder parts); gamma of the synthesis,
      // <dQ(X), Q(X)> with the synthesis' own fp32 output (the training
      // backward's qx32 holds the bf16 Q(X) that the later passes' scores took)
      const float* qx_syn = a.exact ? reinterpret_cast<const float*>(ws + bp.fwd.off_qx32) : qx32;
      if ((st = lat_sum(B, H, M, D, bp.S, 0, sc, gathered, nullptr, R, stride, dqxdec, qx_syn, gsyn, dqx32, s)) !=
              FLARE_OK ||
          (st = pad(q32, q0pad, static_cast<long>(H) * M, D, a.exact ? 1.f : c, s)) != FLARE_OK ||
          (st = pad(dqx32, dqxpad, BH * M, D, 1.f, s)) != FLARE_OK)
        return st;
      // eq. 8 backward with dQ(X) as the upstream gradient: dK~, dV~ rows ...
      TokParams tp = tok_params(B, H, N, M, D, 0, a.lengths, sc, a.sh);
      tp.qpad = q0pad; tp.dzpad = dqxpad; tp.lm = lsyn; tp.gam = gsyn;
      tp.k = kt; tp.v = vt;
      tp.ghi = ghi; tp.glo = glo; tp.g_ld = 4 * C; tp.g_col_k = 2 * C; tp.g_col_v = 3 * C;
      if (use_lat_tc(a.exact, D)) {  // both passes on tcgen05, from the parts of dQ(X)
        if ((st = split_hilo(bp, ws, dqx32, BH * M * D, s)) != FLARE_OK ||
            (st = tok_tc(kTokTcEncoder, bp, ws, kt, vt, nullptr, a.Q0, 0, nullptr, nullptr, lsyn, gsyn, ghi, glo, 4 * C,
                         2 * C, 3 * C, nullptr, nullptr, B, H, N, M, D, a.lengths, sc, s)) != FLARE_OK)
          return st;
        return lat_tc(kLatTcEncoder, bp, ws, a.Q0, 0, ws + bp.off_xhi16, ws + bp.off_xlo16, kt, vt, nullptr, nullptr,
                      lsyn, gsyn, exch, nullptr, B, H, N, M, D, a.lengths, sc, s);
      }
      if (a.exact) tp.smul = c;
      if (launch_tok(kTokEncoder, tp, s) != cudaSuccess) return FLARE_ERR_LAUNCH;
      // ... and the partials of dQ0
      LatParams le = lat_params(bp, ws, q32, 0, kt, B, H, N, M, D, a.lengths, sc, a.sh);
      le.zrow = dqx32; le.lrow = lsyn; le.grow = gsyn; le.v = vt;
      if (a.exact) exact_scores(le, sc);
      le.part_b = exch;
      return launch_lat(kLatEncoder, le, s) == cudaSuccess ? FLARE_OK : FLARE_ERR_LAUNCH;
    }
    case 5: {
      // dQ0, summed over the batch and the shards
      if ((st = lat_sum(B, H, M, D, bp.S, 1, sc, gathered, nullptr, R, stride, nullptr, nullptr, nullptr, a.dQ0, s)) !=
          FLARE_OK)
        return st;
      // projections backward on this shard's rows (tcgen05): dX = G [Wk | Wv | Wk~ | Wv~]^T and the
      // split partials of (X^T G)^T
      const long rows = static_cast<long>(B) * N;
      const CUtensorMapSwizzle sw128 = CU_TENSOR_MAP_SWIZZLE_128B;
      const flare_bf16* w4[4] = {a.Wk, a.Wv, a.Wk_syn, a.Wv_syn};
      DxTcMaps xm;
      DwTcMaps wm;
      if (!map2d(&xm.ghi, ghi, 4 * C, rows, 64, 128, sw128) || !map2d(&xm.glo, glo, 4 * C, rows, 64, 128, sw128) ||
          !map2d(&wm.ghi, ghi, 4 * C, rows, 64, 32, sw128) || !map2d(&wm.glo, glo, 4 * C, rows, 64, 32, sw128) ||
          !map2d(&wm.x, a.X, C, rows, 64, 32, sw128))
        return FLARE_ERR_LAUNCH;
      for (int i = 0; i < 4; ++i)
        if (!map2d(&xm.w[i], w4[i], C, C, 64, C, sw128)) return FLARE_ERR_LAUNCH;
      uint32_t* err = reinterpret_cast<uint32_t*>(ws + bp.fwd.off_err);
      DxTcParams dx{};
      dx.R = static_cast<int>(rows); dx.C = C;
      dx.dx = reinterpret_cast<uint16_t*>(a.dX);
      dx.err = err; dx.timeout_ns = wait_timeout_ns();
      if (launch_dx_tc(xm, dx, s) != cudaSuccess) return FLARE_ERR_LAUNCH;
      DwTcParams dw{};
      dw.R = static_cast<int>(rows); dw.C = C; dw.n_splits = bp.dw_splits; dw.rows_per_split = kBwdDwRows;
      dw.part = exch;
      dw.err = err; dw.timeout_ns = wait_timeout_ns();
      return launch_dw_tc(wm, dw, s) == cudaSuccess ? FLARE_OK : FLARE_ERR_LAUNCH;
    }
    case 6: {
      // dW: the partials of every shard's rows (rank-major, so the splits of all
      // shards form one ascending sequence)
      DwReduceParams dr{};
      dr.C = C; dr.J = 4 * C; dr.n_splits = R * bp.dw_splits; dr.shared = shared ? 1 : 0;
      dr.part = gathered;
      dr.dw[0] = a.dWk; dr.dw[1] = a.dWv; dr.dw[2] = a.dWk_syn; dr.dw[3] = a.dWv_syn;
      return launch_dw_tc_reduce(dr, s) == cudaSuccess ? FLARE_OK : FLARE_ERR_LAUNCH;
    }
    default:
      return FLARE_ERR_SHAPE;
  }
}

flare_status check_bwd_sizes(int B, int H, int N, int M, int D) {
  flare_status st = check_common(B, H, N, M, D);
  if (st != FLARE_OK) return st;
  return static_cast<long>(B) * H > 65535 ? FLARE_ERR_UNSUPPORTED : FLARE_OK;
}

// Checks shared by the FLARE backward entry points.
flare_status check_fl_bwd(const FlArgs& a, const void* workspace) {
  if (!a.K || !a.V || !a.Q || !a.dY || !a.dK || !a.dV || !a.dQ || !workspace) return FLARE_ERR_NULL;
  flare_status st = check_bwd_sizes(a.B, a.H, a.N, a.M, a.D);
  if (st != FLARE_OK) return st;
  if (!aligned16(a.K) || !aligned16(a.V) || !aligned16(a.Q) || !aligned16(a.dY) || !aligned16(a.dK) ||
      !aligned16(a.dV) || !aligned16(a.dQ) || !aligned16(a.lengths) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return FLARE_ERR_ALIGN;
  return FLARE_OK;
}

// Checks shared by the FLARE++ backward entry points.
flare_status check_pp_bwd(const PpArgs& a, const void* workspace) {
  flare_status st = check_flarepp(a.X, a.Wk, a.Wv, a.Wk_syn, a.Wv_syn, a.Q0, a.dY, a.B, a.N, a.C, a.H, a.M, a.D,
                                  a.lengths, workspace, nullptr, nullptr);
  if (st != FLARE_OK) return st;
  const bool shared = a.Wk_syn == a.Wk && a.Wv_syn == a.Wv;
  if (!a.dX || !a.dWk || !a.dWv || !a.dQ0 || (!shared && (!a.dWk_syn || !a.dWv_syn))) return FLARE_ERR_NULL;
  if ((st = check_bwd_sizes(a.B, a.H, a.N, a.M, a.D)) != FLARE_OK) return st;
  if (static_cast<long>(a.B) * a.N > 65535L * kBwdDwRows) return FLARE_ERR_UNSUPPORTED;
  if (!aligned16(a.dX) || !aligned16(a.dWk) || !aligned16(a.dWv) || !aligned16(a.dWk_syn) || !aligned16(a.dWv_syn) ||
      !aligned16(a.dQ0))
    return FLARE_ERR_ALIGN;
  return FLARE_OK;
}

}  // namespace
}  // namespace flare

using namespace flare;

namespace {
// The training pair's launch sequences (defined with the training entry
// points below); the single-GPU backward runs them back to back.
flare_status pp_train_forward(const BwdPlan& bp, uint8_t* ws, const PpArgs& a, flare_bf16* Y, cudaStream_t s);
flare_status pp_train_backward(const BwdPlan& bp, uint8_t* ws, const PpArgs& a, bool check_state, cudaStream_t s);
flare_status fl_train_forward(const BwdPlan& bp, uint8_t* ws, const FlArgs& a, flare_bf16* Y, size_t workspace_bytes,
                              cudaStream_t s);
flare_status fl_train_backward(const BwdPlan& bp, uint8_t* ws, const FlArgs& a, bool check_state, cudaStream_t s);

}  // namespace

extern "C" {

flare_status flare_mixer_bwd(const flare_bf16* K, const flare_bf16* V, const flare_bf16* Q, const flare_bf16* dY,
                             flare_bf16* dK, flare_bf16* dV, float* dQ, int B, int H, int N, int M, int D,
                             const int32_t* lengths, float scale, void* workspace, size_t workspace_bytes,
                             void* stream) {
  FlArgs a{K, V, Q, dY, dK, dV, dQ, B, H, N, M, D, lengths, resolve_scale(scale, D), Shard{0, N, 1}};
  a.exact = true;
  flare_status st = check_fl_bwd(a, workspace);
  if (st != FLARE_OK) return st;
  const BwdPlan bp = make_bwd_plan(false, B, H, N, M, D, 0);
  if (workspace_bytes < bp.total) return FLARE_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  // the statistics come from the forward kernels (a training forward that
  // stores no Y), then the training backward's launches
  if ((st = fl_train_forward(bp, ws, a, nullptr, workspace_bytes, s)) != FLARE_OK) return st;
  return fl_train_backward(bp, ws, a, false, s);
}

size_t flare_cp_bwd_exchange_bytes(int phase, int B, int H, int N, int M, int D) {
  if (phase < 0 || phase >= kFlPhases - 1) return 0;
  if (check_bwd_sizes(B, H, N, M, D) != FLARE_OK) return 0;
  return fl_exchange_floats(make_bwd_plan(false, B, H, N, M, D, 0), phase, B, H, M, D) * sizeof(float);
}

flare_status flare_cp_bwd_phase(int phase, const flare_bf16* K, const flare_bf16* V, const flare_bf16* Q,
                                const flare_bf16* dY, const float* gathered, float* exchange, flare_bf16* dK,
                                flare_bf16* dV, float* dQ, int B, int H, int N, int M, int D, const int32_t* lengths,
                                int rank, int world, float scale, void* workspace, size_t workspace_bytes,
                                void* stream) {
  if (phase < 0 || phase >= kFlPhases) return FLARE_ERR_SHAPE;
  if (world < 1 || rank < 0 || rank >= world) return FLARE_ERR_SHAPE;
  if (static_cast<long>(N) * world >= (1L << 31)) return FLARE_ERR_UNSUPPORTED;
  if ((phase > 0 && !gathered) || (phase < kFlPhases - 1 && !exchange)) return FLARE_ERR_NULL;
  if (!aligned16(gathered) || !aligned16(exchange)) return FLARE_ERR_ALIGN;
  const FlArgs a{K, V, Q, dY, dK, dV, dQ, B, H, N, M, D, lengths, resolve_scale(scale, D),
                 Shard{rank * N, world * N, world}};
  flare_status st = check_fl_bwd(a, workspace);
  if (st != FLARE_OK) return st;
  const BwdPlan bp = make_bwd_plan(false, B, H, N, M, D, 0);
  if (workspace_bytes < bp.total) return FLARE_ERR_WORKSPACE;
  return fl_phase(phase, bp, static_cast<uint8_t*>(workspace), a, gathered, exchange,
                  static_cast<cudaStream_t>(stream));
}

flare_status flarepp_mixer_bwd(const flare_bf16* X, const flare_bf16* Wk, const flare_bf16* Wv,
                               const flare_bf16* Wk_syn, const flare_bf16* Wv_syn, const flare_bf16* Q0,
                               const flare_bf16* dY, flare_bf16* dX, float* dWk, float* dWv, float* dWk_syn,
                               float* dWv_syn, float* dQ0, int B, int N, int C, int H, int M, int D,
                               const int32_t* lengths, float scale, void* workspace, size_t workspace_bytes,
                               void* stream) {
  PpArgs a{X, Wk, Wv, Wk_syn, Wv_syn, Q0, dY, dX, dWk, dWv, dWk_syn, dWv_syn, dQ0,
           B, N, C, H, M, D, lengths, resolve_scale(scale, D), Shard{0, N, 1}};
  a.exact = true;
  flare_status st = check_pp_bwd(a, workspace);
  if (st != FLARE_OK) return st;
  const BwdPlan bp = make_bwd_plan(true, B, H, N, M, D, C);
  if (workspace_bytes < bp.total) return FLARE_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  // the projections, Q(X), Z and the statistics come from the forward
  // kernels (a training forward that stores no Y), then the training
  // backward's launches
  if ((st = pp_train_forward(bp, ws, a, nullptr, s)) != FLARE_OK) return st;
  return pp_train_backward(bp, ws, a, false, s);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Training pair: a forward that keeps, in the backward's workspace, what the
// backward would otherwise recompute (the projections, Q(X) and Z, and the
// log-normalisers of the synthesis and encode softmaxes), and the backward
// that uses it.  The backward's scores then take the bf16 Q(X) that the
// forward's products used, unscaled, with the scale applied to the fp32
// product (exact scores), so that the forward's normalisers fit them.  The
// decoder's delta_n = <dY_n, Y_n> needs Y from the fp32 Z (a Y from the bf16
// Z moves the gradients of Q0 and W~_K by more than the tolerance): at D = 16
// the training forward's decoder adds the low bf16 part of Z and keeps the
// fp32 Y and the per-token normalisers L_n; at D = 32 (no shared memory for
// the low part) the backward recomputes L_n and delta_n.
// ---------------------------------------------------------------------------
namespace {

// What a training forward keeps besides the synthesis normalisers.
FwdStats train_stats(const BwdPlan& bp, uint8_t* ws, int D) {
  FwdStats fs;
  fs.lenc = reinterpret_cast<float*>(ws + bp.off_lenc);
  if (D == 16) {
    fs.zf16 = reinterpret_cast<uint16_t*>(ws + bp.off_zf16);
    fs.y32 = reinterpret_cast<float*>(ws + bp.off_y32);
    fs.ltok = reinterpret_cast<float*>(ws + bp.off_ltok);
  }
  return fs;
}

flare_status set_train_mark(uint8_t* ws, const BwdPlan& bp, int value, cudaStream_t s) {
  return cudaMemsetAsync(ws + bp.fwd.off_err + kTrainMarkOffset, value, 4, s) == cudaSuccess ? FLARE_OK
                                                                                             : FLARE_ERR_LAUNCH;
}

flare_status widen(const uint16_t* src, float* dst, long n, cudaStream_t s) {
  const CvtParams cv{n, src, dst};
  return launch_cvt(cv, s) == cudaSuccess ? FLARE_OK : FLARE_ERR_LAUNCH;
}

// Start of a training backward: clear the error word (not the mark), check
// the mark on the device (check_state; not when the state comes from this
// call's own forward, whose error word is kept), take Q0 (or Q) and Q(X) as
// fp32 images of their bf16 values and the forward's fp32 Z, and pad them
// unscaled.
flare_status train_prologue(const BwdPlan& bp, uint8_t* ws, const flare_bf16* Q, const uint16_t* qx16, long BH, int H,
                            int M, int D, bool check_state, cudaStream_t s) {
  if (check_state) {
    if (cudaMemsetAsync(ws + bp.fwd.off_err, 0, kErrWordBytes, s) != cudaSuccess) return FLARE_ERR_LAUNCH;
    const MarkParams mk{reinterpret_cast<const uint32_t*>(ws + bp.fwd.off_err + kTrainMarkOffset),
                        reinterpret_cast<uint32_t*>(ws + bp.fwd.off_err)};
    if (launch_check_mark(mk, s) != cudaSuccess) return FLARE_ERR_LAUNCH;
  }
  float* q32 = reinterpret_cast<float*>(ws + bp.off_q32);
  float* z32 = reinterpret_cast<float*>(ws + bp.off_z32);
  const size_t lat = static_cast<size_t>(BH) * M * D;
  flare_status st;
  if ((st = widen(reinterpret_cast<const uint16_t*>(Q), q32, static_cast<long>(H) * M * D, s)) != FLARE_OK) return st;
  if (cudaMemcpyAsync(z32, ws + bp.fwd.off_z32, lat * 4, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return FLARE_ERR_LAUNCH;
  const float* qdec = q32;  // FLARE: the learned queries
  if (qx16 != nullptr) {
    float* qx32 = reinterpret_cast<float*>(ws + bp.off_qx32);
    if ((st = widen(qx16, qx32, static_cast<long>(lat), s)) != FLARE_OK) return st;
    qdec = qx32;
  }
  const long qrows = qx16 != nullptr ? BH * M : static_cast<long>(H) * M;
  if ((st = pad(qdec, reinterpret_cast<float*>(ws + bp.off_qpad), qrows, D, 1.f, s)) != FLARE_OK) return st;
  if (use_lat_tc(true, D) && (st = split_hilo(bp, ws, z32, static_cast<long>(lat), s, true)) != FLARE_OK) return st;
  return pad(z32, reinterpret_cast<float*>(ws + bp.off_zpad), BH * M, D, 1.f, s);
}

// The decoder's statistics (L_n, delta_n: from the training forward at
// D = 16, recomputed otherwise) and its backward (the dZ and dQ partials into
// `exch`), exact scores; q: the fp32 queries of the lat pass.
flare_status train_decoder(const BwdPlan& bp, uint8_t* ws, const float* q, const void* q16, int q_per_batch,
                           const void* k, const flare_bf16* dY, int B, int H, int N, int M, int D,
                           const int32_t* lengths, float sc, float* exch, cudaStream_t s) {
  const Shard sh{0, N, 1};
  float* ltok = reinterpret_cast<float*>(ws + bp.off_ltok);
  float* dtok = reinterpret_cast<float*>(ws + bp.off_dtok);
  if (D == 16) {  // L_n is the forward's; delta_n from its fp32 Y
    DeltaParams dp{};
    dp.B = B; dp.H = H; dp.N = N; dp.D = D;
    dp.tok_offset = 0; dp.n_global = N;
    dp.lengths = lengths;
    dp.y32 = reinterpret_cast<const float*>(ws + bp.off_y32);
    dp.dy = reinterpret_cast<const uint16_t*>(dY);
    dp.dtok = dtok;
    if (launch_delta(dp, s) != cudaSuccess) return FLARE_ERR_LAUNCH;
  } else {
    TokParams tp = tok_params(B, H, N, M, D, q_per_batch, lengths, sc, sh);
    tp.smul = sc * kLog2e;
    tp.qpad = reinterpret_cast<const float*>(ws + bp.off_qpad);
    tp.zpad = reinterpret_cast<const float*>(ws + bp.off_zpad);
    tp.k = static_cast<const uint16_t*>(k);
    tp.dy = reinterpret_cast<const uint16_t*>(dY);
    tp.ltok = ltok; tp.dtok = dtok;
    if (launch_tok(kTokStats, tp, s) != cudaSuccess) return FLARE_ERR_LAUNCH;
  }
  const size_t P = part_floats(bp, B, H, M, D, false);
  // Z as the high and low bf16 parts of the fp32 Z; the per-token L_n and
  // delta_n rows go through fp32 tensor maps, whose row stride (4N bytes)
  // must be a multiple of 16
  if (use_lat_tc(true, D) && N % 4 == 0) {
    return lat_tc(kLatTcDecoder, bp, ws, q16, q_per_batch, ws + bp.off_zhi16, ws + bp.off_zlo16, k, dY, ltok, dtok,
                  nullptr, nullptr, exch + P, exch, B, H, N, M, D, lengths, sc, s);
  }
  LatParams ld = lat_params(bp, ws, q, q_per_batch, k, B, H, N, M, D, lengths, sc, sh);
  exact_scores(ld, sc);
  ld.zrow = reinterpret_cast<const float*>(ws + bp.off_z32);
  ld.dy = reinterpret_cast<const uint16_t*>(dY);
  ld.ltok = ltok; ld.dtok = dtok;
  ld.part_a = exch;
  ld.part_b = exch + P;
  return launch_lat(kLatDecoder, ld, s) == cudaSuccess ? FLARE_OK : FLARE_ERR_LAUNCH;
}

// The training forward's launches (FLARE++): the mixer forward that also
// keeps the backward's state; Y may be null (not stored).
flare_status pp_train_forward(const BwdPlan& bp, uint8_t* ws, const PpArgs& a, flare_bf16* Y, cudaStream_t s) {
  FwdStats fs = train_stats(bp, ws, a.D);
  fs.lsyn = reinterpret_cast<float*>(ws + bp.off_lsyn);
  return flarepp_run(bp.fwd, a.X, a.Wk, a.Wv, a.Wk_syn, a.Wv_syn, a.Q0, Y, 0, a.B, a.N, a.C, a.H, a.M, a.D,
                     a.lengths, a.sc, ws, s, nullptr, nullptr, nullptr, nullptr, &fs);
}

// The training backward's launches after the argument checks (FLARE++).
flare_status pp_train_backward(const BwdPlan& bp, uint8_t* ws, const PpArgs& a, bool check_state, cudaStream_t s) {
  const long BH = static_cast<long>(a.B) * a.H;
  float* pa = reinterpret_cast<float*>(ws + bp.off_pa);
  float* pc = reinterpret_cast<float*>(ws + bp.off_pc);
  flare_status st;
  if ((st = train_prologue(bp, ws, a.Q0, reinterpret_cast<const uint16_t*>(ws + bp.fwd.off_qx16), BH, a.H, a.M, a.D,
                           check_state, s)) != FLARE_OK ||
      (st = train_decoder(bp, ws, reinterpret_cast<const float*>(ws + bp.off_qx32), ws + bp.fwd.off_qx16, 1,
                          ws + bp.fwd.off_kp, a.dY, a.B, a.H, a.N, a.M, a.D, a.lengths, a.sc, pa, s)) != FLARE_OK)
    return st;
  // phases 3-6 of the seven (the exchanges stay in the workspace)
  float* ex[kPpPhases - 1] = {nullptr, nullptr, pa, pc, pc, reinterpret_cast<float*>(ws + bp.off_dwpart)};
  for (int ph = 3; ph < kPpPhases; ++ph)
    if ((st = pp_phase(ph, bp, ws, a, ex[ph - 1], ph < kPpPhases - 1 ? ex[ph] : nullptr, s)) != FLARE_OK) return st;
  return FLARE_OK;
}

// The training forward's launches (FLARE); Y may be null (not stored).
flare_status fl_train_forward(const BwdPlan& bp, uint8_t* ws, const FlArgs& a, flare_bf16* Y, size_t workspace_bytes,
                              cudaStream_t s) {
  FwdStats fs = train_stats(bp, ws, a.D);
  return flare_fwd(a.K, a.V, a.Q, Y, a.B, a.H, a.N, a.M, a.D, a.lengths, a.sc, ws, workspace_bytes, s, nullptr,
                   nullptr, nullptr, &fs);
}

// The training backward's launches after the argument checks (FLARE).
flare_status fl_train_backward(const BwdPlan& bp, uint8_t* ws, const FlArgs& a, bool check_state, cudaStream_t s) {
  float* pa = reinterpret_cast<float*>(ws + bp.off_pa);
  float* pc = reinterpret_cast<float*>(ws + bp.off_pc);
  flare_status st;
  if ((st = train_prologue(bp, ws, a.Q, nullptr, static_cast<long>(a.B) * a.H, a.H, a.M, a.D, check_state, s)) !=
          FLARE_OK ||
      (st = train_decoder(bp, ws, reinterpret_cast<const float*>(ws + bp.off_q32), a.Q, 0, a.K, a.dY, a.B, a.H, a.N,
                          a.M, a.D, a.lengths, a.sc, pa, s)) != FLARE_OK ||
      (st = fl_phase(2, bp, ws, a, pa, pc, s)) != FLARE_OK || (st = fl_phase(3, bp, ws, a, pc, nullptr, s)) != FLARE_OK)
    return st;
  return FLARE_OK;
}

}  // namespace

extern "C" {

flare_status flarepp_mixer_fwd_train(const flare_bf16* X, const flare_bf16* Wk, const flare_bf16* Wv,
                                     const flare_bf16* Wk_syn, const flare_bf16* Wv_syn, const flare_bf16* Q0,
                                     flare_bf16* Y, int B, int N, int C, int H, int M, int D, const int32_t* lengths,
                                     float scale, void* workspace, size_t workspace_bytes, void* stream) {
  flare_status st = check_flarepp(X, Wk, Wv, Wk_syn, Wv_syn, Q0, Y, B, N, C, H, M, D, lengths, workspace, nullptr,
                                  nullptr);
  if (st != FLARE_OK) return st;
  if ((st = check_bwd_sizes(B, H, N, M, D)) != FLARE_OK) return st;
  const BwdPlan bp = make_bwd_plan(true, B, H, N, M, D, C);
  if (workspace_bytes < bp.total) return FLARE_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const PpArgs a{X, Wk, Wv, Wk_syn, Wv_syn, Q0, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                 B, N, C, H, M, D, lengths, resolve_scale(scale, D), Shard{0, N, 1}};
  if ((st = pp_train_forward(bp, ws, a, Y, s)) != FLARE_OK) return st;
  return set_train_mark(ws, bp, kTrainStateByte, s);
}

flare_status flarepp_mixer_bwd_train(const flare_bf16* X, const flare_bf16* Wk, const flare_bf16* Wv,
                                     const flare_bf16* Wk_syn, const flare_bf16* Wv_syn, const flare_bf16* Q0,
                                     const flare_bf16* dY, flare_bf16* dX, float* dWk, float* dWv, float* dWk_syn,
                                     float* dWv_syn, float* dQ0, int B, int N, int C, int H, int M, int D,
                                     const int32_t* lengths, float scale, void* workspace, size_t workspace_bytes,
                                     void* stream) {
  PpArgs a{X, Wk, Wv, Wk_syn, Wv_syn, Q0, dY, dX, dWk, dWv, dWk_syn, dWv_syn, dQ0,
           B, N, C, H, M, D, lengths, resolve_scale(scale, D), Shard{0, N, 1}};
  a.exact = true;
  flare_status st = check_pp_bwd(a, workspace);
  if (st != FLARE_OK) return st;
  const BwdPlan bp = make_bwd_plan(true, B, H, N, M, D, C);
  if (workspace_bytes < bp.total) return FLARE_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  if ((st = pp_train_backward(bp, ws, a, true, s)) != FLARE_OK) return st;
  return set_train_mark(ws, bp, 0, s);  // the state is used: a second backward needs a new forward
}

flare_status flare_mixer_fwd_train(const flare_bf16* K, const flare_bf16* V, const flare_bf16* Q, flare_bf16* Y,
                                   int B, int H, int N, int M, int D, const int32_t* lengths, float scale,
                                   void* workspace, size_t workspace_bytes, void* stream) {
  if (!K || !V || !Q || !Y || !workspace) return FLARE_ERR_NULL;
  flare_status st = check_bwd_sizes(B, H, N, M, D);
  if (st != FLARE_OK) return st;
  const BwdPlan bp = make_bwd_plan(false, B, H, N, M, D, 0);
  if (workspace_bytes < bp.total) return FLARE_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const FlArgs a{K, V, Q, nullptr, nullptr, nullptr, nullptr, B, H, N, M, D, lengths, resolve_scale(scale, D),
                 Shard{0, N, 1}};
  if ((st = fl_train_forward(bp, ws, a, Y, workspace_bytes, s)) != FLARE_OK) return st;
  return set_train_mark(ws, bp, kTrainStateByte, s);
}

flare_status flare_mixer_bwd_train(const flare_bf16* K, const flare_bf16* V, const flare_bf16* Q, const flare_bf16* dY,
                                   flare_bf16* dK, flare_bf16* dV, float* dQ, int B, int H, int N, int M, int D,
                                   const int32_t* lengths, float scale, void* workspace, size_t workspace_bytes,
                                   void* stream) {
  FlArgs a{K, V, Q, dY, dK, dV, dQ, B, H, N, M, D, lengths, resolve_scale(scale, D), Shard{0, N, 1}};
  a.exact = true;
  flare_status st = check_fl_bwd(a, workspace);
  if (st != FLARE_OK) return st;
  const BwdPlan bp = make_bwd_plan(false, B, H, N, M, D, 0);
  if (workspace_bytes < bp.total) return FLARE_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  if ((st = fl_train_backward(bp, ws, a, true, s)) != FLARE_OK) return st;
  return set_train_mark(ws, bp, 0, s);
}

size_t flarepp_cp_bwd_exchange_bytes(int phase, int B, int N, int C, int H, int M, int D) {
  if (phase < 0 || phase >= kPpPhases - 1) return 0;
  if (check_bwd_sizes(B, H, N, M, D) != FLARE_OK || C != H * D || C % 64 != 0 || C > 256) return 0;
  return pp_exchange_floats(make_bwd_plan(true, B, H, N, M, D, C), phase, B, H, M, D, C) * sizeof(float);
}

flare_status flarepp_cp_bwd_phase(int phase, const flare_bf16* X, const flare_bf16* Wk, const flare_bf16* Wv,
                                  const flare_bf16* Wk_syn, const flare_bf16* Wv_syn, const flare_bf16* Q0,
                                  const flare_bf16* dY, const float* gathered, float* exchange, flare_bf16* dX,
                                  float* dWk, float* dWv, float* dWk_syn, float* dWv_syn, float* dQ0, int B, int N,
                                  int C, int H, int M, int D, const int32_t* lengths, int rank, int world,
                                  float scale, void* workspace, size_t workspace_bytes, void* stream) {
  if (phase < 0 || phase >= kPpPhases) return FLARE_ERR_SHAPE;
  if (world < 1 || rank < 0 || rank >= world) return FLARE_ERR_SHAPE;
  if (static_cast<long>(N) * world >= (1L << 31)) return FLARE_ERR_UNSUPPORTED;
  if ((phase > 0 && !gathered) || (phase < kPpPhases - 1 && !exchange)) return FLARE_ERR_NULL;
  if (!aligned16(gathered) || !aligned16(exchange)) return FLARE_ERR_ALIGN;
  const PpArgs a{X, Wk, Wv, Wk_syn, Wv_syn, Q0, dY, dX, dWk, dWv, dWk_syn, dWv_syn, dQ0,
                 B, N, C, H, M, D, lengths, resolve_scale(scale, D), Shard{rank * N, world * N, world}};
  flare_status st = check_pp_bwd(a, workspace);
  if (st != FLARE_OK) return st;
  const BwdPlan bp = make_bwd_plan(true, B, H, N, M, D, C);
  if (workspace_bytes < bp.total) return FLARE_ERR_WORKSPACE;
  return pp_phase(phase, bp, static_cast<uint8_t*>(workspace), a, gathered, exchange,
                  static_cast<cudaStream_t>(stream));
}

}  // extern "C"
