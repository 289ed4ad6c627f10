// Latent-parallel backward passes on tcgen05 (D = 16 or 32): the gradients of the
// encoder softmax with respect to its queries (FLARE++ paper, eq. 8 and 10;
// FLARE paper, eq. 5) and of the decoder softmax with respect to its queries
// and latent values (eq. 11; eq. 6), for the training backward, whose
// queries are bf16 values (Q(X), Q0 or the learned Q) so that the score
// products are exact.  Per head, latent block of 128 rows and token split:
//
//   encoder (kLatTcEncoder), for each token tile:
//     S = Q K^T                         UMMA M=128 (latents) x N=T, fp32 TMEM
//     G = dZ V^T = dZhi V^T + dZlo V^T  two UMMAs (dZ fp32 as two bf16 parts)
//     W = 2^(S c - L_m), dS = W (G - gamma_m)      softmax threads, one row each
//     dQ += dS K = dShi K + dSlo K      TS-form UMMAs, dS from TMEM as bf16 parts
//   decoder (kLatTcDecoder):
//     S = Q K^T, G = Z dY^T (Z as two bf16 parts)
//     W = 2^(S c - L_n), dS = W (G - delta_n)       L_n, delta_n per token column
//     dQ += dS K (two parts), dZ += W dY            TS-form UMMAs
//
// written as split partials [B*H][S][M][D] (dQ; the decoder's dZ as well),
// summed in a fixed order by lat_sum_kernel as the tf32 passes' are.  The
// score scale c = scale log2(e) is applied to the fp32 product, as in the
// forward's kernels, so that the forward's normalisers L_m fit these scores.
//
// Tiles of T = 48 tokens (32 at D = 32) stream through a TMA ring (K and V,
// or K and dY, plus L_n and delta_n for the decoder).  TMEM: S at column 0,
// G at T, dQ at 2T, dZ at 2T + D (128 columns: four CTAs per SM).  The score
// products take K = D in k-steps of 16.  The softmax threads read a
// tile's S and G in three 16-column pieces (the next piece's TMEM load in
// flight while the current one is computed) and write, over the piece they
// have read, dS as bf16 high and low parts (S columns [16j, 16j+8) and
// [16j+8, 16j+16)) and, for the decoder, W in bf16 (G columns [16j, 16j+8)):
// each 16-token k-step of the value MMAs then takes its A operand from 8
// consecutive columns.  One score buffer: the MMA thread issues the next
// tile's S and G once the value MMAs of the previous tile are done; the four
// co-resident CTAs of an SM fill each other's gaps.
//
// Warp roles (5 warps): warp 0 lane 0 issues the TMA loads and the MMAs;
// warps 1..4 are the softmax warps (thread <-> TMEM lane <-> latent row).
#include "bwd_internal.h"
#include "ptx.cuh"

namespace flare {
namespace {

// After tcgen05.wait::ld: the registers a TMEM load wrote are defined here,
// so that no use of them is scheduled before the wait.
__device__ __forceinline__ void regs_defined(uint32_t (&r)[16]) {
  asm volatile(""
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                 "+r"(r[15]));
}

template <int D_>
struct LatTcCfg {
  static constexpr int D = D_;
  static constexpr int T = D == 16 ? 48 : 32;           // tokens per tile
  static constexpr int ROWB = D * 2;                    // bytes of one bf16 row
  static constexpr int TILE_B = T * ROWB;               // one K, V or dY tile
  static constexpr int ROWS_B = kLatBlock * ROWB;       // Q, or one part of dZ / Z
  static constexpr int LD_B = 256;                      // one tile's L_n or delta_n (T floats, padded)
  static constexpr int NST = 6;                         // ring stages
  static constexpr uint32_t LAYOUT = D == 16 ? LAYOUT_SW32 : LAYOUT_SW64;
  static constexpr uint32_t SBO = 8 * ROWB;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_XA = OFF_Q + ROWS_B;         // dZhi (encoder) or Zhi (decoder)
  static constexpr int OFF_XB = OFF_XA + ROWS_B;        // the low parts
  static constexpr int OFF_K = OFF_XB + ROWS_B;         // NST x K tile
  static constexpr int OFF_U = OFF_K + NST * TILE_B;    // NST x (V or dY) tile
  static constexpr int OFF_LD = OFF_U + NST * TILE_B;   // NST x (L_n | delta_n)
  static constexpr int OFF_BAR = OFF_LD + NST * 2 * LD_B;
  static constexpr int OFF_MISC = OFF_BAR + 8 * (6 + NST);
  static constexpr int BYTES = OFF_MISC + 64 + NST * 4;
  static constexpr uint32_t COL_S = 0, COL_G = T, COL_DQ = 2 * T, COL_DZ = 2 * T + D;
  static constexpr uint32_t TMEM_COLS = 128;
  static constexpr int THREADS = 160;
  static constexpr int CTAS_PER_SM = 4;
  static_assert(COL_DZ + D <= TMEM_COLS, "TMEM columns");
  static_assert(TILE_B % (8 * ROWB) == 0 && ROWS_B % 1024 == 0, "tiles must hold whole swizzle atoms");
  static_assert(T % 16 == 0 && T * 4 <= LD_B, "tile of L_n / delta_n");
};

template <int MODE, int DD>
__global__ void __launch_bounds__(LatTcCfg<DD>::THREADS, LatTcCfg<DD>::CTAS_PER_SM)
    lat_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_xa,
                  const __grid_constant__ CUtensorMap tm_xb, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_u, const __grid_constant__ CUtensorMap tm_l,
                  const __grid_constant__ CUtensorMap tm_d, const LatTcParams p) {
  using Cfg = LatTcCfg<DD>;
  constexpr int D = Cfg::D, T = Cfg::T, NST = Cfg::NST;
  constexpr bool DEC = MODE == kLatTcDecoder;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sq = sm + Cfg::OFF_Q;
  uint8_t* sxa = sm + Cfg::OFF_XA;
  uint8_t* sxb = sm + Cfg::OFF_XB;
  uint8_t* sk = sm + Cfg::OFF_K;
  uint8_t* su = sm + Cfg::OFF_U;
  uint8_t* sld = sm + Cfg::OFF_LD;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Cfg::OFF_BAR);
  uint64_t* q_full = bars;                 // Q and both parts of dZ / Z landed
  uint64_t* s_full = bars + 1;             // S and G of the current tile computed
  uint64_t* p_full = bars + 2;             // dS (and W) stored by every softmax warp
  uint64_t* pv_done = bars + 3;            // the value MMAs of the tile done
  uint64_t* o_full = bars + 4;             // every MMA of the CTA done
  uint64_t* kv_full = bars + 6;            // [NST] ring stage landed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + Cfg::OFF_MISC);
  int* abort_flag = reinterpret_cast<int*>(sm + Cfg::OFF_MISC + 4);
  volatile int* last_load = reinterpret_cast<volatile int*>(sm + Cfg::OFF_MISC + 64);  // per stage

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int LB = p.n_lblocks, S = p.n_splits;
  const int lb = blockIdx.x % LB;
  const int s = (blockIdx.x / LB) % S;
  const int bh = blockIdx.x / (LB * S);
  const int b = bh / p.H, h = bh % p.H;
  const int g = p.q_per_batch ? bh : h;
  bool bad_len = false;
  const int L = shard_valid_len(p.lengths, b, p.N, 0, p.N, &bad_len);
  if (bad_len && threadIdx.x == 0) atomicOr(p.err, FLARE_DEV_BAD_LENGTH);
  // this split's tokens [n_begin, n_end), in tiles of T
  const int n_begin = s * p.split_tokens;
  const int n_end = min(n_begin + p.split_tokens, L);
  const int ntiles = n_end > n_begin ? (n_end - n_begin + T - 1) / T : 0;
  const size_t part_row0 = (static_cast<size_t>(bh) * S + s) * p.M;
  pdl_launch_dependents();

  if (ntiles == 0) {  // empty split: zero partials
    pdl_wait();
    for (int i = threadIdx.x; i < kLatBlock * D; i += blockDim.x) {
      const int m = lb * kLatBlock + i / D;
      if (m < p.M) {
        p.part_q[(part_row0 + m) * D + i % D] = 0.f;
        if (DEC) p.part_z[(part_row0 + m) * D + i % D] = 0.f;
      }
    }
    return;
  }

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(s_full, 1);
    mbar_init(p_full, 4);
    mbar_init(pv_done, 1);
    mbar_init(o_full, 1);
    for (int i = 0; i < NST; ++i) {
      mbar_init(kv_full + i, 1);
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
  // tile n of the split into ring stage n % NST (one thread)
  auto load_tile = [&](int n) {
    const int st = n % NST;
    const int tok = n_begin + n * T;
    mbar_arrive_expect_tx(kv_full + st, 2 * Cfg::TILE_B + (DEC ? 2 * T * 4 : 0));
    tma_load_3d(sk + st * Cfg::TILE_B, &tm_k, kv_full + st, 0, tok, bh);
    tma_load_3d(su + st * Cfg::TILE_B, &tm_u, kv_full + st, 0, tok, bh);
    if (DEC) {
      tma_load_2d(sld + st * 2 * Cfg::LD_B, &tm_l, kv_full + st, tok, bh);
      tma_load_2d(sld + st * 2 * Cfg::LD_B + Cfg::LD_B, &tm_d, kv_full + st, tok, bh);
    }
    last_load[st] = n;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ MMA thread
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_xa);
      tma_prefetch_desc(&tm_xb);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_u);
      mbar_arrive_expect_tx(q_full, 3 * p.q_rows * Cfg::ROWB);
      tma_load_3d(sq, &tm_q, q_full, 0, lb * kLatBlock, g);
      tma_load_3d(sxa, &tm_xa, q_full, 0, lb * kLatBlock, bh);
      tma_load_3d(sxb, &tm_xb, q_full, 0, lb * kLatBlock, bh);
      for (int n = 0; n < min(NST, ntiles); ++n) load_tile(n);
      const uint32_t idesc_s = idesc_bf16_f32(128, T, false, false);
      const uint32_t idesc_v = idesc_bf16_f32(128, D, false, true);
      const uint64_t q_desc = umma_desc(smem_u32(sq), 16, Cfg::SBO, Cfg::LAYOUT);
      const uint64_t xa_desc = umma_desc(smem_u32(sxa), 16, Cfg::SBO, Cfg::LAYOUT);
      const uint64_t xb_desc = umma_desc(smem_u32(sxb), 16, Cfg::SBO, Cfg::LAYOUT);
      // a ring tile as the K-major B operand of a score product (N = T
      // tokens) and as the MN-major B operand of a value product (N = D,
      // k-steps of 16 tokens); a stage's descriptor adds its offset >> 4
      const uint64_t k_desc = umma_desc(smem_u32(sk), 16, Cfg::SBO, Cfg::LAYOUT);
      const uint64_t u_desc = umma_desc(smem_u32(su), 16, Cfg::SBO, Cfg::LAYOUT);
      constexpr uint64_t STAGE = Cfg::TILE_B >> 4, KSTEP = (16 * Cfg::ROWB) >> 4;
      bool ok = mbar_wait_mma(q_full, 0, wc);
      for (int i = 0; ok && i < ntiles; ++i) {
        const int st = i % NST;
        if (i > 0) {
          // the value MMAs of tile i - 1 are done: S and G may be overwritten,
          // and tile i - 1's stage takes tile i - 1 + NST
          if (!mbar_wait_mma(pv_done, (i - 1) & 1, wc)) { ok = false; break; }
          if (i - 1 + NST < ntiles) load_tile(i - 1 + NST);
        }
        if (!mbar_wait_mma(kv_full + st, (i / NST) & 1, wc)) { ok = false; break; }
        tc_fence_after();
        const uint64_t kd = k_desc + st * STAGE, ud = u_desc + st * STAGE;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {  // k-steps of 16 along D: 32 bytes inside the row
          const uint64_t ko = 2 * kk;
          umma_ss(tmem + Cfg::COL_S, q_desc + ko, kd + ko, idesc_s, kk > 0 ? 1u : 0u);
          umma_ss(tmem + Cfg::COL_G, xa_desc + ko, ud + ko, idesc_s, kk > 0 ? 1u : 0u);
          umma_ss(tmem + Cfg::COL_G, xb_desc + ko, ud + ko, idesc_s, 1u);
        }
        umma_commit(s_full);
        if (!mbar_wait_mma(p_full, i & 1, wc)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < T / 16; ++ks) {
          const uint32_t a = tmem + Cfg::COL_S + 16 * ks;
          umma_ts(tmem + Cfg::COL_DQ, a, kd + ks * KSTEP, idesc_v, (i > 0 || ks > 0) ? 1u : 0u);  // dShi K
          umma_ts(tmem + Cfg::COL_DQ, a + 8, kd + ks * KSTEP, idesc_v, 1u);                      // dSlo K
          if (DEC)
            umma_ts(tmem + Cfg::COL_DZ, tmem + Cfg::COL_G + 16 * ks, ud + ks * KSTEP, idesc_v,
                    (i > 0 || ks > 0) ? 1u : 0u);                                                // W dY
        }
        umma_commit(pv_done);
      }
      umma_commit(o_full);  // completes once every MMA issued above is done
      mbar_wait_drain(o_full, 0, p.timeout_ns);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int wq = warp & 3;                  // TMEM lane quarter of this warp
    const int r = wq * 32 + lane;             // latent row within the block
    const int m = lb * kLatBlock + r;
    const bool row_ok = m < p.M;
    const bool warp_live = lb * kLatBlock + wq * 32 < p.M;
    const float c = p.c;
    // encoder: the row's normaliser and gamma
    float lrow = 0.f, grow = 0.f;
    if (!DEC && row_ok) {
      lrow = p.lrow[static_cast<size_t>(bh) * p.M + m];
      grow = p.grow[static_cast<size_t>(bh) * p.M + m];
    }
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    // One 16-column piece: scores s and products g (raw fp32 bits), for the
    // decoder its tokens' L_n at ld[0..16) and delta_n at ld[LD_B/4 ..); dS =
    // W (g - delta) with W = 2^(s c - L) out as bf16 high and low parts (and
    // W in bf16).  Pairs of columns go through the paired fp32x2 forms.
    const uint64_t c2 = f2_pack(c, c), m1 = f2_pack(-1.f, -1.f), zero2 = f2_pack(0.f, 0.f);
    const uint64_t neg_l2 = f2_pack(-lrow, -lrow), neg_g2 = f2_pack(-grow, -grow);
    auto piece = [&](const uint32_t (&sp)[16], const uint32_t (&gp)[16], const float* ld, uint32_t (&hi)[8],
                     uint32_t (&lo)[8], uint32_t (&wp)[8]) {
      float4 lq = make_float4(0.f, 0.f, 0.f, 0.f), dq = lq;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint64_t s2 = f2_pack(__uint_as_float(sp[2 * k]), __uint_as_float(sp[2 * k + 1]));
        const uint64_t g2 = f2_pack(__uint_as_float(gp[2 * k]), __uint_as_float(gp[2 * k + 1]));
        uint64_t t2, e2;
        if (DEC) {  // L_n, delta_n of the pair's token columns (shared-memory broadcast, four at a time)
          if ((k & 1) == 0) {
            lq = *reinterpret_cast<const float4*>(ld + 2 * k);
            dq = *reinterpret_cast<const float4*>(ld + Cfg::LD_B / 4 + 2 * k);
          }
          const uint64_t l2 = (k & 1) ? f2_pack(lq.z, lq.w) : f2_pack(lq.x, lq.y);
          const uint64_t d2 = (k & 1) ? f2_pack(dq.z, dq.w) : f2_pack(dq.x, dq.y);
          t2 = f2_fma(l2, m1, f2_fma(s2, c2, zero2));   // s c - L_n
          e2 = f2_fma(d2, m1, g2);                       // g - delta_n
        } else {
          t2 = f2_fma(s2, c2, neg_l2);                   // s c - L_m
          e2 = f2_add(g2, neg_g2);                       // g - gamma_m
        }
        float t0, t1;
        f2_unpack(t2, t0, t1);
        const float w0 = ex2_mufu(t0), w1 = ex2_mufu(t1);
        const uint64_t d2 = f2_fma(f2_pack(w0, w1), e2, zero2);  // dS = W (g - .)
        float d0, d1;
        f2_unpack(d2, d0, d1);
        hi[k] = pack_bf16x2(d0, d1);
        float r0, r1;
        f2_unpack(f2_fma(f2_pack(bf16_lo(hi[k]), bf16_hi(hi[k])), m1, d2), r0, r1);  // dS - hi
        lo[k] = pack_bf16x2(r0, r1);
        if (DEC) wp[k] = pack_bf16x2(w0, w1);
      }
    };
    bool ok = true;
    for (int i = 0; i < ntiles; ++i) {
      if (!mbar_wait_warp(s_full, i & 1, wc)) { ok = false; break; }
      tc_fence_after();
      const int valid = min(T, n_end - (n_begin + i * T));
      const float* sl = reinterpret_cast<const float*>(sld + (i % NST) * 2 * Cfg::LD_B);
      if (warp_live) {
        const bool full = valid >= T;  // every token column of the tile is valid
        uint32_t sv[2][16], gv[2][16];
        tmem_ld16(lane_base + Cfg::COL_S, sv[0]);
        tmem_ld16(lane_base + Cfg::COL_G, gv[0]);
        tmem_wait_ld();
        regs_defined(sv[0]);
        regs_defined(gv[0]);
#pragma unroll
        for (int j = 0; j < T / 16; ++j) {
          uint32_t hi[8], lo[8], wp[8];
          const int cb = j & 1, nb = cb ^ 1;
          if (j + 1 < T / 16) {  // the next piece, while this one is computed
            tmem_ld16(lane_base + Cfg::COL_S + 16 * (j + 1), sv[nb]);
            tmem_ld16(lane_base + Cfg::COL_G + 16 * (j + 1), gv[nb]);
          }
          piece(sv[cb], gv[cb], sl + 16 * j, hi, lo, wp);
          if (!full) {  // the tile's last valid token column is in this tile: zero the columns past it
            const int nv = valid - 16 * j;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const uint32_t keep = 2 * k + 1 < nv ? 0xFFFFFFFFu : 2 * k < nv ? 0x0000FFFFu : 0u;
              hi[k] &= keep;
              lo[k] &= keep;
              wp[k] &= keep;
            }
          }
          // over the 16 columns just read: dS high and low parts (and W)
          tmem_st8(lane_base + Cfg::COL_S + 16 * j, hi);
          tmem_st8(lane_base + Cfg::COL_S + 16 * j + 8, lo);
          if (DEC) tmem_st8(lane_base + Cfg::COL_G + 16 * j, wp);
          if (j + 1 < T / 16) {
            tmem_wait_ld();
            regs_defined(sv[nb]);
            regs_defined(gv[nb]);
          }
        }
        tmem_wait_st();
      }
      tc_fence_before();
      mbar_arrive_warp(p_full);
      __syncwarp();
    }
    if (ok && mbar_wait_warp(o_full, 0, wc)) {
      tc_fence_after();
      if (warp_live) {
        uint32_t dq[D], dz[D];
        tmem_ld_cols<D>(lane_base + Cfg::COL_DQ, dq);
        if (DEC) tmem_ld_cols<D>(lane_base + Cfg::COL_DZ, dz);
        tmem_wait_ld();
        if (row_ok) {
          float4* oq = reinterpret_cast<float4*>(p.part_q + (part_row0 + m) * D);
#pragma unroll
          for (int u = 0; u < D / 4; ++u)
            oq[u] = make_float4(__uint_as_float(dq[4 * u]), __uint_as_float(dq[4 * u + 1]),
                                __uint_as_float(dq[4 * u + 2]), __uint_as_float(dq[4 * u + 3]));
          if (DEC) {
            float4* oz = reinterpret_cast<float4*>(p.part_z + (part_row0 + m) * D);
#pragma unroll
            for (int u = 0; u < D / 4; ++u)
              oz[u] = make_float4(__uint_as_float(dz[4 * u]), __uint_as_float(dz[4 * u + 1]),
                                  __uint_as_float(dz[4 * u + 2]), __uint_as_float(dz[4 * u + 3]));
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    if (lane == 0) {  // copies still in flight (only after an abort) must land before exit
      for (int st = 0; st < NST; ++st)
        if (last_load[st] >= 0) mbar_wait_drain(kv_full + st, (last_load[st] / NST) & 1, p.timeout_ns);
      mbar_wait_drain(q_full, 0, p.timeout_ns);
    }
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::TMEM_COLS);
  }
}

__global__ void __launch_bounds__(256) split_hilo_kernel(const SplitHiLoParams p) {
  const long i = 2 * (static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x);
  if (i >= p.n) return;
  const float2 x = *reinterpret_cast<const float2*>(p.x + i);
  const uint32_t h = pack_bf16x2(x.x, x.y);
  *reinterpret_cast<uint32_t*>(p.hi + i) = h;
  *reinterpret_cast<uint32_t*>(p.lo + i) = pack_bf16x2(x.x - bf16_lo(h), x.y - bf16_hi(h));
}

}  // namespace

cudaError_t launch_split_hilo(const SplitHiLoParams& p, cudaStream_t s) {
  const long pairs = p.n / 2;
  split_hilo_kernel<<<static_cast<unsigned>((pairs + 255) / 256), 256, 0, s>>>(p);
  return cudaGetLastError();
}

size_t lat_tc_smem_bytes(int D) {
  const size_t need = (D == 16 ? LatTcCfg<16>::BYTES : LatTcCfg<32>::BYTES) + 1024;
  // at most CTAS_PER_SM CTAs per SM (228 KB each, 1 KB of it reserved per
  // CTA), so that every resident CTA finds its TMEM columns free
  const size_t floor = (228 * 1024) / (LatTcCfg<16>::CTAS_PER_SM + 1) + 1024;
  return need > floor ? need : floor;
}

int lat_tc_tile(int D) { return D == 16 ? LatTcCfg<16>::T : LatTcCfg<32>::T; }

cudaError_t launch_lat_tc(int mode, const LatTcMaps& m, const LatTcParams& p, cudaStream_t s) {
  if (p.D != 16 && p.D != 32) return cudaErrorInvalidValue;
  const size_t smem = lat_tc_smem_bytes(p.D);
  const dim3 grid(static_cast<unsigned>(p.B * p.H * p.n_lblocks * p.n_splits));
  auto go = [&](auto kern) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    kern<<<grid, LatTcCfg<16>::THREADS, smem, s>>>(m.q, m.xa, m.xb, m.k, m.u, mode == kLatTcDecoder ? m.l : m.k,
                                                   mode == kLatTcDecoder ? m.d : m.k, p);
    return cudaGetLastError();
  };
  if (p.D == 16)
    return mode == kLatTcDecoder ? go(lat_tc_kernel<kLatTcDecoder, 16>) : go(lat_tc_kernel<kLatTcEncoder, 16>);
  return mode == kLatTcDecoder ? go(lat_tc_kernel<kLatTcDecoder, 32>) : go(lat_tc_kernel<kLatTcEncoder, 32>);
}

}  // namespace flare
