// Token-parallel backward passes on tcgen05 (D = 16 or 32): the gradients of the
// key and value rows for the training backward, whose queries are bf16
// values (Q(X), Q0 or the learned Q) so that the score products are exact.
// One CTA owns a tile of 128 tokens of one head (thread <-> TMEM lane <->
// token) and walks the latents in chunks of C = 16 (full) or 48 (encoder
// only; 32 at D = 32):
//
//   full (kTokTcFull: decoder and encoder, FLARE++ paper eq. 10-11; FLARE
//   paper eq. 5-6), per chunk:
//     S = K Q_c^T, dA = V dZ_c^T, dP = dY Z_c^T     UMMA M=128 x N=C, fp32 TMEM
//       (dZ and Z fp32, each as two bf16 parts: two UMMAs)
//     A = 2^(S c - L_m), P = 2^(S c - L_n)
//     dS = A (dA - gamma_m) + P (dP - delta_n)       softmax threads
//     dK += dS Q_c (two bf16 parts of dS), dV += A dZ_c (two parts of dZ)
//   encoder only (kTokTcEncoder: the query synthesis, eq. 8, with dQ(X) in
//   the place of dZ): the A terms alone.
//
// dK is scaled by scale = ln 2 * (scale log2 e) in the epilogue; rows of
// padding tokens are zero.  The score scale is applied to the fp32 product,
// as in the forward, so that the forward's normalisers L_m fit these scores.
//
// The token tile's K, V and dY stay in shared memory; the latents (Q, the
// parts of Z and dZ, L_m and gamma_m) stream through a TMA ring (stages of 32
// latents, two chunks, in the full pass; of one 48-latent chunk in the
// encoder-only one).  The dK, dV accumulators sit at TMEM columns 128 - 2D
// and 128 - D (128 columns: four CTAs per SM).  Full pass at D = 16: two
// score buffers (S, dA, dP:
// 16 columns each); the MMA thread issues chunk j + 1's score products into
// the other buffer before it waits for the softmax threads to finish chunk
// j, so the score products of one chunk overlap the softmax of the previous
// one (measured: 4.39 against 5.02 ms per million-token launch with one
// buffer of 32-latent chunks).  Encoder-only pass: one buffer (S at 0, dA at
// 48), read in 16-column pieces, the next chunk's products issued once the
// value products of the previous one are done (with half the work per
// score, two buffers of 16-latent chunks measured slower: 3.64 against 3.36
// ms).  At D = 32 the accumulators take 64 columns, which leaves room for
// one score buffer: 16-latent chunks for the full pass, 32 for the encoder
// only.  The score products take K = D in k-steps of 16.  The softmax
// threads write, over each 16-column piece they have read,
// dS as bf16 high and low parts (S columns [0, 8) and [8, 16) of the piece)
// and A in bf16 (dA columns [0, 8)); the value MMAs take them as TMEM A
// operands, one 16-latent k-step per piece.
//
// Warp roles (5 warps): warp 0 lane 0 issues the TMA loads and the MMAs;
// warps 1..4 are the softmax warps.
#include "bwd_internal.h"
#include "ptx.cuh"

namespace flare {
namespace {

__device__ __forceinline__ void regs_defined16(uint32_t (&r)[16]) {
  asm volatile(""
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                 "+r"(r[15]));
}

template <int MODE, int D_>
struct TokTcCfg {
  static constexpr bool FULL = MODE == kTokTcFull;
  static constexpr int D = D_;
  static constexpr bool DB = FULL && D == 16;           // two score buffers
  static constexpr int C = FULL ? 16 : (D == 16 ? 48 : 32);  // latents per chunk
  static constexpr int CR = DB ? 2 * C : C;             // latents per ring stage
  static constexpr int CPS = CR / C;                    // chunks per ring stage
  static constexpr int TT = kBwdTokBlock;               // tokens per CTA (128)
  static constexpr int ROWB = D * 2;
  static constexpr int TOK_B = TT * ROWB;               // one token tile (K, V or dY)
  static constexpr int CH_B = CR * ROWB;                // a stage's rows of Q, Zhi, Zlo, dZhi or dZlo
  static constexpr int NCH = FULL ? 5 : 3;              // latent tensors per ring stage
  static constexpr int ST_B = NCH * CH_B + 2 * 256;     // a ring stage: the tensors, L_m, gamma_m
  static constexpr int NST = D == 16 ? 6 : 4;
  static constexpr uint32_t LAYOUT = D == 16 ? LAYOUT_SW32 : LAYOUT_SW64;
  static constexpr uint32_t SBO = 8 * ROWB;
  static constexpr int OFF_TK = 0, OFF_TV = TOK_B, OFF_TY = 2 * TOK_B;
  static constexpr int OFF_RING = (FULL ? 3 : 2) * TOK_B;
  // within a stage
  static constexpr int S_Q = 0, S_DH = CH_B, S_DL = 2 * CH_B, S_ZH = 3 * CH_B, S_ZL = 4 * CH_B;
  static constexpr int S_LM = NCH * CH_B, S_GM = NCH * CH_B + 256;
  static constexpr int OFF_BAR = OFF_RING + NST * ST_B;
  static constexpr int OFF_MISC = OFF_BAR + 8 * (8 + NST);
  static constexpr int BYTES = OFF_MISC + 64 + NST * 4;
  // one score buffer: S, dA (and dP) of a chunk
  static constexpr uint32_t BUF = FULL ? 3 * C : 2 * C;
  static constexpr int NBUF = DB ? 2 : 1;
  static constexpr uint32_t COL_S = 0, COL_DA = C, COL_DP = 2 * C, COL_DK = 128 - 2 * D, COL_DV = 128 - D;
  static constexpr uint32_t TMEM_COLS = 128;
  static constexpr int THREADS = 160;
  static constexpr int CTAS_PER_SM = 4;
  static_assert(COL_DV + D <= TMEM_COLS && NBUF * BUF <= COL_DK, "TMEM columns");
  static_assert(TOK_B % 1024 == 0 && CH_B % (8 * ROWB) == 0 && ST_B % 256 == 0 && (C * ROWB) % (8 * ROWB) == 0,
                "tiles and chunks must hold whole swizzle atoms");
  static_assert(CR * 4 <= 256, "L_m / gamma_m of a stage");
};

template <int MODE, int DD>
__global__ void __launch_bounds__(TokTcCfg<MODE, DD>::THREADS, TokTcCfg<MODE, DD>::CTAS_PER_SM)
    tok_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                  const __grid_constant__ CUtensorMap tm_y, const __grid_constant__ CUtensorMap tm_q,
                  const __grid_constant__ CUtensorMap tm_zh, const __grid_constant__ CUtensorMap tm_zl,
                  const __grid_constant__ CUtensorMap tm_dh, const __grid_constant__ CUtensorMap tm_dl,
                  const __grid_constant__ CUtensorMap tm_lm, const __grid_constant__ CUtensorMap tm_gm,
                  const TokTcParams p) {
  using Cfg = TokTcCfg<MODE, DD>;
  constexpr int D = Cfg::D, C = Cfg::C, NST = Cfg::NST;
  constexpr bool FULL = MODE == kTokTcFull;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stk = sm + Cfg::OFF_TK;
  uint8_t* stv = sm + Cfg::OFF_TV;
  uint8_t* sty = sm + Cfg::OFF_TY;
  uint8_t* ring = sm + Cfg::OFF_RING;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Cfg::OFF_BAR);
  uint64_t* tok_full = bars;               // the token tile landed
  uint64_t* s_full = bars + 1;             // [2] a buffer's S, dA (dP) computed
  uint64_t* p_full = bars + 3;             // [2] dS and A of a buffer stored by every softmax warp
  uint64_t* pv_done = bars + 5;            // [2] a buffer's value MMAs done
  uint64_t* o_full = bars + 7;             // every MMA of the CTA done
  uint64_t* lat_full = bars + 8;           // [NST] ring stage landed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + Cfg::OFF_MISC);
  int* abort_flag = reinterpret_cast<int*>(sm + Cfg::OFF_MISC + 4);
  volatile int* last_load = reinterpret_cast<volatile int*>(sm + Cfg::OFF_MISC + 64);  // per stage

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles = (p.N + Cfg::TT - 1) / Cfg::TT;
  const int tile = blockIdx.x % tiles;
  const int bh = blockIdx.x / tiles;
  const int b = bh / p.H, h = bh % p.H;
  const int g = p.q_per_batch ? bh : h;
  bool bad_len = false;
  const int L = shard_valid_len(p.lengths, b, p.N, 0, p.N, &bad_len);
  if (bad_len && threadIdx.x == 0) atomicOr(p.err, FLARE_DEV_BAD_LENGTH);
  const int n0 = tile * Cfg::TT;
  const int nchunks = (p.M + C - 1) / C;   // M is a multiple of 16: so is a last partial chunk
  const int nstages = (p.M + Cfg::CR - 1) / Cfg::CR;
  pdl_launch_dependents();

  // one token row of the outputs (zeros for padding tokens)
  auto store_row = [&](int n, const float (&dk)[D], const float (&dv)[D]) {
    if (p.ghi != nullptr) {  // high and low bf16 parts of the fp32 rows
      const size_t o = (static_cast<size_t>(b) * p.N + n) * p.g_ld + h * D;
      auto put = [&](int col, const float (&x)[D]) {
        uint32_t hi[D / 2], lo[D / 2];
#pragma unroll
        for (int k = 0; k < D / 2; ++k) {
          hi[k] = pack_bf16x2(x[2 * k], x[2 * k + 1]);
          lo[k] = pack_bf16x2(x[2 * k] - bf16_lo(hi[k]), x[2 * k + 1] - bf16_hi(hi[k]));
        }
        uint4* dh = reinterpret_cast<uint4*>(p.ghi + o + col);
        uint4* dl = reinterpret_cast<uint4*>(p.glo + o + col);
#pragma unroll
        for (int u = 0; u < D / 8; ++u) {
          dh[u] = make_uint4(hi[4 * u], hi[4 * u + 1], hi[4 * u + 2], hi[4 * u + 3]);
          dl[u] = make_uint4(lo[4 * u], lo[4 * u + 1], lo[4 * u + 2], lo[4 * u + 3]);
        }
      };
      put(p.g_col_k, dk);
      put(p.g_col_v, dv);
    } else {
      uint4* ok = reinterpret_cast<uint4*>(p.dk16 + (static_cast<size_t>(bh) * p.N + n) * D);
      uint4* ov = reinterpret_cast<uint4*>(p.dv16 + (static_cast<size_t>(bh) * p.N + n) * D);
#pragma unroll
      for (int u = 0; u < D / 8; ++u) {
        ok[u] = make_uint4(pack_bf16x2(dk[8 * u], dk[8 * u + 1]), pack_bf16x2(dk[8 * u + 2], dk[8 * u + 3]),
                           pack_bf16x2(dk[8 * u + 4], dk[8 * u + 5]), pack_bf16x2(dk[8 * u + 6], dk[8 * u + 7]));
        ov[u] = make_uint4(pack_bf16x2(dv[8 * u], dv[8 * u + 1]), pack_bf16x2(dv[8 * u + 2], dv[8 * u + 3]),
                           pack_bf16x2(dv[8 * u + 4], dv[8 * u + 5]), pack_bf16x2(dv[8 * u + 6], dv[8 * u + 7]));
      }
    }
  };

  if (n0 >= L) {  // every token of the tile is padding: zero rows
    pdl_wait();
    float zero[D];
#pragma unroll
    for (int d = 0; d < D; ++d) zero[d] = 0.f;
    for (int r = threadIdx.x; r < Cfg::TT; r += blockDim.x)
      if (n0 + r < p.N) store_row(n0 + r, zero, zero);
    return;
  }

  if (threadIdx.x == 0) {
    mbar_init(tok_full, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(s_full + b, 1);
      mbar_init(p_full + b, 4);
      mbar_init(pv_done + b, 1);
    }
    mbar_init(o_full, 1);
    for (int i = 0; i < NST; ++i) {
      mbar_init(lat_full + i, 1);
      last_load[i] = -1;
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx wc{p.err, abort_flag, p.timeout_ns};
  // latents [32 j, 32 j + 32) into ring stage j % NST (one thread)
  auto load_stage = [&](int j) {
    const int st = j % NST, m0 = j * Cfg::CR;
    uint8_t* sb = ring + st * Cfg::ST_B;
    mbar_arrive_expect_tx(lat_full + st, (FULL ? 5 : 3) * Cfg::CH_B + 2 * Cfg::CR * 4);
    tma_load_3d(sb + Cfg::S_Q, &tm_q, lat_full + st, 0, m0, g);
    tma_load_3d(sb + Cfg::S_DH, &tm_dh, lat_full + st, 0, m0, bh);
    tma_load_3d(sb + Cfg::S_DL, &tm_dl, lat_full + st, 0, m0, bh);
    if (FULL) {
      tma_load_3d(sb + Cfg::S_ZH, &tm_zh, lat_full + st, 0, m0, bh);
      tma_load_3d(sb + Cfg::S_ZL, &tm_zl, lat_full + st, 0, m0, bh);
    }
    tma_load_2d(sb + Cfg::S_LM, &tm_lm, lat_full + st, m0, bh);
    tma_load_2d(sb + Cfg::S_GM, &tm_gm, lat_full + st, m0, bh);
    last_load[st] = j;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ MMA thread
    if (lane == 0) {
      mbar_arrive_expect_tx(tok_full, (FULL ? 3 : 2) * Cfg::TOK_B);
      tma_load_3d(stk, &tm_k, tok_full, 0, n0, bh);
      tma_load_3d(stv, &tm_v, tok_full, 0, n0, bh);
      if (FULL) tma_load_3d(sty, &tm_y, tok_full, 0, n0, bh);
      for (int j = 0; j < min(NST, nstages); ++j) load_stage(j);
      const uint32_t idesc_v = idesc_bf16_f32(128, D, false, true);
      const uint32_t idesc_s = idesc_bf16_f32(128, C, false, false);
      const uint64_t tk_desc = umma_desc(smem_u32(stk), 16, Cfg::SBO, Cfg::LAYOUT);
      const uint64_t tv_desc = umma_desc(smem_u32(stv), 16, Cfg::SBO, Cfg::LAYOUT);
      const uint64_t ty_desc = umma_desc(smem_u32(sty), 16, Cfg::SBO, Cfg::LAYOUT);
      // a chunk as the K-major B operand of a score product (N = C latents)
      // and as the MN-major B operand of a value product (N = D, k-steps of
      // 16 latents); a chunk's descriptor adds its offset >> 4
      const uint64_t r_desc = umma_desc(smem_u32(ring), 16, Cfg::SBO, Cfg::LAYOUT);
      constexpr uint64_t STAGE = Cfg::ST_B >> 4, HALF = (Cfg::C * Cfg::ROWB) >> 4;
      constexpr uint64_t OQ = Cfg::S_Q >> 4, OZH = Cfg::S_ZH >> 4, OZL = Cfg::S_ZL >> 4, ODH = Cfg::S_DH >> 4,
                         ODL = Cfg::S_DL >> 4;
      constexpr int CPS = Cfg::CPS;
      // S = K Q_c^T, dA = V dZ_c^T (two parts) and, full, dP = dY Z_c^T (two
      // parts) into the buffer at tb; K = D in k-steps of 16 (32 bytes inside
      // the rows)
      auto score_products = [&](uint32_t tb, uint64_t rd, uint32_t idesc) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t ko = 2 * kk;
          const uint32_t a0 = kk > 0 ? 1u : 0u;
          umma_ss(tb + Cfg::COL_S, tk_desc + ko, rd + OQ + ko, idesc, a0);
          umma_ss(tb + Cfg::COL_DA, tv_desc + ko, rd + ODH + ko, idesc, a0);
          umma_ss(tb + Cfg::COL_DA, tv_desc + ko, rd + ODL + ko, idesc, 1u);
          if (FULL) {
            umma_ss(tb + Cfg::COL_DP, ty_desc + ko, rd + OZH + ko, idesc, a0);
            umma_ss(tb + Cfg::COL_DP, ty_desc + ko, rd + OZL + ko, idesc, 1u);
          }
        }
      };
      auto chunk_desc = [&](int j) { return r_desc + ((j / CPS) % NST) * STAGE + (j % CPS) * HALF; };
      bool ok = mbar_wait_mma(tok_full, 0, wc);
      if constexpr (Cfg::DB) {
        // the score products of chunk j into buffer j & 1
        auto scores = [&](int j) -> bool {
          const int sj = j / CPS;
          if (!mbar_wait_mma(lat_full + sj % NST, (sj / NST) & 1, wc)) return false;
          tc_fence_after();
          const uint64_t rd = chunk_desc(j);
          const uint32_t tb = tmem + (j & 1) * Cfg::BUF;
          score_products(tb, rd, idesc_s);
          umma_commit(s_full + (j & 1));
          return true;
        };
        ok = ok && scores(0);
        for (int j = 0; ok && j < nchunks; ++j) {
          if (j + 1 < nchunks) {
            if (j >= 1) {
              // chunk j - 1's value MMAs are done: its buffer takes chunk
              // j + 1, and once every chunk of a stage is done the stage is
              // refilled
              if (!mbar_wait_mma(pv_done + ((j - 1) & 1), ((j - 1) >> 1) & 1, wc)) { ok = false; break; }
              if ((j - 1) % CPS == CPS - 1 && (j - 1) / CPS + NST < nstages) load_stage((j - 1) / CPS + NST);
            }
            if (!scores(j + 1)) { ok = false; break; }
          }
          if (!mbar_wait_mma(p_full + (j & 1), (j >> 1) & 1, wc)) { ok = false; break; }
          tc_fence_after();
          const uint64_t rd = chunk_desc(j);
          const uint32_t tb = tmem + (j & 1) * Cfg::BUF;
          const uint32_t acc0 = j > 0 ? 1u : 0u;
          umma_ts(tmem + Cfg::COL_DK, tb + Cfg::COL_S, rd + OQ, idesc_v, acc0);        // dShi Q_c
          umma_ts(tmem + Cfg::COL_DK, tb + Cfg::COL_S + 8, rd + OQ, idesc_v, 1u);      // dSlo Q_c
          umma_ts(tmem + Cfg::COL_DV, tb + Cfg::COL_DA, rd + ODH, idesc_v, acc0);      // A dZhi_c
          umma_ts(tmem + Cfg::COL_DV, tb + Cfg::COL_DA, rd + ODL, idesc_v, 1u);        // A dZlo_c
          umma_commit(pv_done + (j & 1));
        }
      } else {
        constexpr uint64_t KSTEP = (16 * Cfg::ROWB) >> 4;
        for (int j = 0; ok && j < nchunks; ++j) {
          const int st = j % NST;
          const int cn = min(C, p.M - j * C);  // C, or a multiple of 16 for the last chunk
          if (j > 0) {
            // the value MMAs of chunk j - 1 are done: S and dA may be
            // overwritten, and its ring stage takes chunk j - 1 + NST
            if (!mbar_wait_mma(pv_done, (j - 1) & 1, wc)) { ok = false; break; }
            if (j - 1 + NST < nstages) load_stage(j - 1 + NST);
          }
          if (!mbar_wait_mma(lat_full + st, (j / NST) & 1, wc)) { ok = false; break; }
          tc_fence_after();
          const uint64_t rd = chunk_desc(j);
          const uint32_t idesc_c = idesc_bf16_f32(128, cn, false, false);
          score_products(tmem, rd, idesc_c);
          umma_commit(s_full);
          if (!mbar_wait_mma(p_full, j & 1, wc)) { ok = false; break; }
          tc_fence_after();
          for (int ks = 0; ks < cn / 16; ++ks) {
            const uint32_t as = tmem + Cfg::COL_S + 16 * ks, aa = tmem + Cfg::COL_DA + 16 * ks;
            const uint32_t acc0 = (j > 0 || ks > 0) ? 1u : 0u;
            umma_ts(tmem + Cfg::COL_DK, as, rd + OQ + ks * KSTEP, idesc_v, acc0);       // dShi Q_c
            umma_ts(tmem + Cfg::COL_DK, as + 8, rd + OQ + ks * KSTEP, idesc_v, 1u);     // dSlo Q_c
            umma_ts(tmem + Cfg::COL_DV, aa, rd + ODH + ks * KSTEP, idesc_v, acc0);      // A dZhi_c
            umma_ts(tmem + Cfg::COL_DV, aa, rd + ODL + ks * KSTEP, idesc_v, 1u);        // A dZlo_c
          }
          umma_commit(pv_done);
        }
      }
      umma_commit(o_full);  // completes once every MMA issued above is done
      mbar_wait_drain(o_full, 0, p.timeout_ns);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int wq = warp & 3;
    const int r = wq * 32 + lane;             // token row within the tile
    const int n = n0 + r;
    const bool tok_ok = n < L;
    const float c = p.c;
    // the decoder's per-token normaliser and delta
    float ln = 0.f, dl = 0.f;
    if (FULL && tok_ok) {
      ln = p.ltok[static_cast<size_t>(bh) * p.N + n];
      dl = p.dtok[static_cast<size_t>(bh) * p.N + n];
    }
    const uint64_t c2 = f2_pack(c, c), m1 = f2_pack(-1.f, -1.f), zero2 = f2_pack(0.f, 0.f);
    const uint64_t neg_ln2 = f2_pack(-ln, -ln), neg_dl2 = f2_pack(-dl, -dl);
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    // one 16-column piece: dS = A (dA - gamma) + P (dP - delta) as bf16 high
    // and low parts, A in bf16
    auto piece = [&](const uint32_t (&sp)[16], const uint32_t (&ap)[16], const uint32_t (&pp)[16], const float* lm,
                     const float* gm, uint32_t (&hi)[8], uint32_t (&lo)[8], uint32_t (&wa)[8]) {
      float4 lq = make_float4(0.f, 0.f, 0.f, 0.f), gq = lq;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        if ((k & 1) == 0) {  // L_m, gamma_m of four latent columns (shared-memory broadcast)
          lq = *reinterpret_cast<const float4*>(lm + 2 * k);
          gq = *reinterpret_cast<const float4*>(gm + 2 * k);
        }
        const uint64_t l2 = (k & 1) ? f2_pack(lq.z, lq.w) : f2_pack(lq.x, lq.y);
        const uint64_t g2 = (k & 1) ? f2_pack(gq.z, gq.w) : f2_pack(gq.x, gq.y);
        const uint64_t s2 = f2_pack(__uint_as_float(sp[2 * k]), __uint_as_float(sp[2 * k + 1]));
        const uint64_t a2 = f2_pack(__uint_as_float(ap[2 * k]), __uint_as_float(ap[2 * k + 1]));
        const uint64_t sc2 = f2_fma(s2, c2, zero2);
        float t0, t1;
        f2_unpack(f2_fma(l2, m1, sc2), t0, t1);  // s c - L_m
        const float w0 = ex2_mufu(t0), w1 = ex2_mufu(t1);
        const uint64_t wa2 = f2_pack(w0, w1);
        uint64_t d2 = f2_fma(wa2, f2_fma(g2, m1, a2), zero2);  // A (dA - gamma_m)
        if (FULL) {
          float u0, u1;
          f2_unpack(f2_add(sc2, neg_ln2), u0, u1);  // s c - L_n
          const uint64_t p2 = f2_pack(ex2_mufu(u0), ex2_mufu(u1));
          const uint64_t q2 = f2_pack(__uint_as_float(pp[2 * k]), __uint_as_float(pp[2 * k + 1]));
          d2 = f2_fma(p2, f2_add(q2, neg_dl2), d2);  // + P (dP - delta_n)
        }
        float d0, d1;
        f2_unpack(d2, d0, d1);
        hi[k] = pack_bf16x2(d0, d1);
        float r0, r1;
        f2_unpack(f2_fma(f2_pack(bf16_lo(hi[k]), bf16_hi(hi[k])), m1, d2), r0, r1);  // dS - hi
        lo[k] = pack_bf16x2(r0, r1);
        wa[k] = pack_bf16x2(w0, w1);
      }
    };
    bool ok = true;
    if constexpr (Cfg::DB) {
      for (int j = 0; j < nchunks; ++j) {
        const int b = j & 1;
        if (!mbar_wait_warp(s_full + b, (j >> 1) & 1, wc)) { ok = false; break; }
        tc_fence_after();
        const uint8_t* sb = ring + ((j / Cfg::CPS) % NST) * Cfg::ST_B;
        const float* lm = reinterpret_cast<const float*>(sb + Cfg::S_LM) + (j % Cfg::CPS) * C;
        const float* gm = reinterpret_cast<const float*>(sb + Cfg::S_GM) + (j % Cfg::CPS) * C;
        const uint32_t tb = lane_base + b * Cfg::BUF;
        uint32_t sv[16], av[16], pv[16], hi[8], lo[8], wa[8];
        tmem_ld16(tb + Cfg::COL_S, sv);
        tmem_ld16(tb + Cfg::COL_DA, av);
        if (FULL) tmem_ld16(tb + Cfg::COL_DP, pv);
        tmem_wait_ld();
        regs_defined16(sv);
        regs_defined16(av);
        if (FULL) regs_defined16(pv);
        piece(sv, av, pv, lm, gm, hi, lo, wa);
        tmem_st8(tb + Cfg::COL_S, hi);
        tmem_st8(tb + Cfg::COL_S + 8, lo);
        tmem_st8(tb + Cfg::COL_DA, wa);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive_warp(p_full + b);
        __syncwarp();
      }
    } else {
      for (int j = 0; j < nchunks; ++j) {
        if (!mbar_wait_warp(s_full, j & 1, wc)) { ok = false; break; }
        tc_fence_after();
        const int cn = min(C, p.M - j * C);
        const uint8_t* sb = ring + (j % NST) * Cfg::ST_B;
        const float* lm = reinterpret_cast<const float*>(sb + Cfg::S_LM);
        const float* gm = reinterpret_cast<const float*>(sb + Cfg::S_GM);
        for (int q = 0; q < cn / 16; ++q) {
          uint32_t sv[16], av[16], pv[16], hi[8], lo[8], wa[8];
          tmem_ld16(lane_base + Cfg::COL_S + 16 * q, sv);
          tmem_ld16(lane_base + Cfg::COL_DA + 16 * q, av);
          if (FULL) tmem_ld16(lane_base + Cfg::COL_DP + 16 * q, pv);
          tmem_wait_ld();
          regs_defined16(sv);
          regs_defined16(av);
          if (FULL) regs_defined16(pv);
          piece(sv, av, pv, lm + 16 * q, gm + 16 * q, hi, lo, wa);
          tmem_st8(lane_base + Cfg::COL_S + 16 * q, hi);
          tmem_st8(lane_base + Cfg::COL_S + 16 * q + 8, lo);
          tmem_st8(lane_base + Cfg::COL_DA + 16 * q, wa);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive_warp(p_full);
        __syncwarp();
      }
    }
    if (ok && mbar_wait_warp(o_full, 0, wc)) {
      tc_fence_after();
      uint32_t kv[D], vv[D];
      tmem_ld_cols<D>(lane_base + Cfg::COL_DK, kv);
      tmem_ld_cols<D>(lane_base + Cfg::COL_DV, vv);
      tmem_wait_ld();
      if (n < p.N) {
        float dk[D], dv[D];
        const float kscale = 0.6931471805599453f * c;  // scale = ln 2 * (scale log2 e)
#pragma unroll
        for (int d = 0; d < D; ++d) {
          dk[d] = tok_ok ? __uint_as_float(kv[d]) * kscale : 0.f;
          dv[d] = tok_ok ? __uint_as_float(vv[d]) : 0.f;
        }
        store_row(n, dk, dv);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    if (lane == 0) {  // copies still in flight (only after an abort) must land before exit
      for (int st = 0; st < NST; ++st)
        if (last_load[st] >= 0) mbar_wait_drain(lat_full + st, (last_load[st] / NST) & 1, p.timeout_ns);
      mbar_wait_drain(tok_full, 0, p.timeout_ns);
    }
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::TMEM_COLS);
  }
}

}  // namespace

template <int MODE, int D>
size_t tok_tc_smem() {
  const size_t need = TokTcCfg<MODE, D>::BYTES + 1024;
  // at most CTAS_PER_SM CTAs per SM (228 KB each, 1 KB of it reserved per
  // CTA), so that every resident CTA finds its TMEM columns free
  const size_t floor = (228 * 1024) / (TokTcCfg<MODE, D>::CTAS_PER_SM + 1) + 1024;
  return need > floor ? need : floor;
}

size_t tok_tc_smem_bytes(int mode, int D) {
  if (D == 16) return mode == kTokTcFull ? tok_tc_smem<kTokTcFull, 16>() : tok_tc_smem<kTokTcEncoder, 16>();
  return mode == kTokTcFull ? tok_tc_smem<kTokTcFull, 32>() : tok_tc_smem<kTokTcEncoder, 32>();
}

int tok_tc_chunk(int mode, int D) {
  if (D == 16) return mode == kTokTcFull ? TokTcCfg<kTokTcFull, 16>::CR : TokTcCfg<kTokTcEncoder, 16>::CR;
  return mode == kTokTcFull ? TokTcCfg<kTokTcFull, 32>::CR : TokTcCfg<kTokTcEncoder, 32>::CR;
}

cudaError_t launch_tok_tc(int mode, const TokTcMaps& m, const TokTcParams& p, cudaStream_t s) {
  if (p.D != 16 && p.D != 32) return cudaErrorInvalidValue;
  const size_t smem = tok_tc_smem_bytes(mode, p.D);
  const int tiles = (p.N + kBwdTokBlock - 1) / kBwdTokBlock;
  const dim3 grid(static_cast<unsigned>(static_cast<long>(p.B) * p.H * tiles));
  auto go = [&](auto kern) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    kern<<<grid, TokTcCfg<kTokTcFull, 16>::THREADS, smem, s>>>(m.k, m.v, m.y, m.q, m.zh, m.zl, m.dh, m.dl, m.lm,
                                                               m.gm, p);
    return cudaGetLastError();
  };
  if (p.D == 16)
    return mode == kTokTcFull ? go(tok_tc_kernel<kTokTcFull, 16>) : go(tok_tc_kernel<kTokTcEncoder, 16>);
  return mode == kTokTcFull ? go(tok_tc_kernel<kTokTcFull, 32>) : go(tok_tc_kernel<kTokTcEncoder, 32>);
}

}  // namespace flare
