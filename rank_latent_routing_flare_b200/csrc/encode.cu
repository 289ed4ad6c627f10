// Split-N encoder SDPA on tcgen05 (FLARE++ paper, arXiv 2608.11519, section
// "Method": the FLARE encoder Z_h = softmax_n(Q_h K_h^T / sqrt(D)) V_h of
// eq. 5, which is also the query synthesis of eq. 8 and the encode of eq. 10).
//
// One CTA owns (b, h, a block of 128 latents, a contiguous range of token
// tiles).  Per 64-token tile:
//   S = Q_blk K_tile^T            UMMA M=128 (latents) x N=64 (tokens), fp32 in TMEM
//   P = 2^(S * c - U_m)           softmax threads, one latent row per thread
//   O += P [V_tile | 1]           UMMA with A = P read from TMEM; the ones block
//                                 makes column D of O the running row sum
// The shift U_m = c * |q_m| * max_{n in split} |k_n| is an upper bound of the
// row's scaled scores (Cauchy-Schwarz), fixed for the whole split, so no
// running maximum and no rescaling of O is needed.  The split writes
// (U_m, sum_m, O_m) and the merge kernel combines splits with the exact
// log-sum-exp rule of section "Multi-GPU context parallelism" (eq. 14).
//
// Warp roles: warp 0 = TMA producer, warp 1 = MMA issuer + TMEM owner,
// warps 2..5 = softmax (thread <-> TMEM lane <-> latent row).
#include "ptx.cuh"

namespace flare {
namespace {

template <int D>
struct EncCfg {
  static constexpr int ROWB = D * 2;                   // bytes of one K/V/Q row
  static constexpr int TILE_B = kEncTile * ROWB;       // bytes of one K or V tile
  static constexpr int Q_B = kLatBlock * ROWB;
  static constexpr int NST = 8;                        // K/V ring stages
  static constexpr uint32_t LAYOUT = (D == 16) ? LAYOUT_SW32 : LAYOUT_SW64;
  static constexpr uint32_t SBO = 8 * ROWB;            // stride of 8-row core-matrix groups
  static constexpr int NO = D + 16;                    // O columns: D values + 16 copies of the sum
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_B;
  static constexpr int OFF_V = OFF_K + NST * TILE_B;
  static constexpr int OFF_ONES = OFF_V + NST * TILE_B;
  static constexpr int OFF_BAR = OFF_ONES + TILE_B;
  static constexpr int OFF_MISC = OFF_BAR + 8 * 32;
  static constexpr int BYTES = OFF_MISC + 64;
  // TMEM columns: S[0..1] at 0 and 64 (fp32 scores), P[0..1] at 128 and 160
  // (bf16 pairs), O at 192 (D values + the row-sum block)
  static constexpr uint32_t TMEM_COLS = 256;
  static constexpr uint32_t COL_S = 0, COL_P = 128, COL_O = 192;
};

template <int D>
__global__ void __launch_bounds__(192, 2)
    encode_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const EncodeParams p) {
  using Cfg = EncCfg<D>;
  constexpr int NST = Cfg::NST;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sq = sm + Cfg::OFF_Q;
  uint8_t* sk = sm + Cfg::OFF_K;
  uint8_t* sv = sm + Cfg::OFF_V;
  uint8_t* sones = sm + Cfg::OFF_ONES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Cfg::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = bars + 1 + NST;
  uint64_t* s_full = bars + 1 + 2 * NST;  // S[j] computed
  uint64_t* s_free = s_full + 2;           // S[j] loaded by the softmax warps
  uint64_t* p_full = s_free + 2;           // P[j] stored by the softmax warps
  uint64_t* p_free = p_full + 2;           // P[j] consumed by the value MMA
  uint64_t* o_full = p_free + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + Cfg::OFF_MISC);
  int* abort_flag = reinterpret_cast<int*>(sm + Cfg::OFF_MISC + 4);
  float* red = reinterpret_cast<float*>(sm + Cfg::OFF_MISC + 16);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int LB = p.n_lblocks, S = p.n_splits;
  const int lb = blockIdx.x % LB;
  const int s = (blockIdx.x / LB) % S;
  const int bh = blockIdx.x / (LB * S);
  const int b = bh / p.H, h = bh % p.H;
  int L = p.N;
  if (p.lengths) {
    int l = p.lengths[b];
    if (l < 1 || l > p.N) {
      if (threadIdx.x == 0) atomicOr(p.err, FLARE_DEV_BAD_LENGTH);
      l = min(max(l, 0), p.N);
    }
    L = l;
  }
  const int ntiles_valid = (L + kEncTile - 1) / kEncTile;
  const int t0 = s * p.tiles_per_split;
  const int t1 = min(t0 + p.tiles_per_split, ntiles_valid);
  const int ntiles = max(0, t1 - t0);
  const int g = p.q_per_batch ? bh : h;
  float* part_base = p.part + static_cast<size_t>(bh * S + s) * p.M * (D + 2);

  if (ntiles == 0) {  // empty split: contributes nothing to the merge
    for (int r = threadIdx.x; r < kLatBlock; r += blockDim.x) {
      const int m = lb * kLatBlock + r;
      if (m < p.M) {
        float* o = part_base + static_cast<size_t>(m) * (D + 2);
        o[0] = -INFINITY;
        o[1] = 0.f;
#pragma unroll
        for (int d = 0; d < D; ++d) o[2 + d] = 0.f;
      }
    }
    return;
  }

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < NST; ++i) {
      mbar_init(kv_full + i, 1);
      mbar_init(kv_empty + i, 1);
    }
    for (int j = 0; j < 2; ++j) {
      mbar_init(s_full + j, 1);
      mbar_init(s_free + j, 128);
      mbar_init(p_full + j, 128);
      mbar_init(p_free + j, 1);
    }
    mbar_init(o_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  for (int i = threadIdx.x; i < Cfg::TILE_B / 4; i += blockDim.x)
    reinterpret_cast<uint32_t*>(sones)[i] = 0x3F803F80u;  // bf16 1.0 pairs
  fence_proxy_async_smem();
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx wc{p.err, abort_flag, p.timeout_ns};

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      mbar_arrive_expect_tx(q_full, p.q_rows * Cfg::ROWB);
      tma_load_3d(sq, &tm_q, q_full, 0, lb * kLatBlock, g);
      int issued = 0;
      for (int i = 0; i < ntiles; ++i) {
        const int st = i % NST;
        if (!mbar_wait(kv_empty + st, ((i / NST) & 1) ^ 1, wc)) break;
        mbar_arrive_expect_tx(kv_full + st, 2 * Cfg::TILE_B);
        const int tok = (t0 + i) * kEncTile;
        tma_load_3d(sk + st * Cfg::TILE_B, &tm_k, kv_full + st, 0, tok, bh);
        tma_load_3d(sv + st * Cfg::TILE_B, &tm_v, kv_full + st, 0, tok, bh);
        issued = i + 1;
      }
      // every issued copy must have landed before the CTA may exit
      for (int i = max(0, issued - NST); i < issued; ++i)
        mbar_wait_drain(kv_full + (i % NST), (i / NST) & 1, p.timeout_ns);
      mbar_wait_drain(q_full, 0, p.timeout_ns);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Order: S(i+2) is issued as soon as the softmax warps have loaded S(i)
    // (early release of the score buffer), then P(i) V(i) once P(i) is in
    // TMEM.  Two score and two probability buffers keep a full tile of slack
    // between the tensor pipe and the softmax warps.
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16_f32(128, kEncTile, false, false);
      const uint32_t idesc_pv = idesc_bf16_f32(128, Cfg::NO, false, true);
      const uint32_t tO = tmem + Cfg::COL_O;
      const uint32_t sq_a = smem_u32(sq);
      const uint32_t ones_a = smem_u32(sones);
      auto issue_s = [&](int i) -> bool {
        const int st = i % NST, j = i & 1;
        if (!mbar_wait(kv_full + st, (i / NST) & 1, wc)) return false;
        if (i >= 2 && !mbar_wait(s_free + j, ((i >> 1) - 1) & 1, wc)) return false;
        tc_fence_after();
        const uint32_t k_a = smem_u32(sk + st * Cfg::TILE_B);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          umma_ss(tmem + Cfg::COL_S + j * 64, umma_desc(sq_a + kk * 32, 16, Cfg::SBO, Cfg::LAYOUT),
                  umma_desc(k_a + kk * 32, 16, Cfg::SBO, Cfg::LAYOUT), idesc_s, kk > 0 ? 1u : 0u);
        }
        umma_commit(s_full + j);
        return true;
      };
      auto issue_pv = [&](int i) -> bool {
        const int j = i & 1, st = i % NST;
        if (!mbar_wait(p_full + j, (i >> 1) & 1, wc)) return false;
        tc_fence_after();
        const uint32_t v_a = smem_u32(sv + st * Cfg::TILE_B);
        const uint32_t lbo = ones_a - v_a;  // [V | 1] : second N-atom = ones block
#pragma unroll
        for (int ks = 0; ks < kEncTile / 16; ++ks) {
          const uint64_t bdesc = umma_desc(v_a + ks * 16 * Cfg::ROWB, lbo, Cfg::SBO, Cfg::LAYOUT);
          umma_ts(tO, tmem + Cfg::COL_P + j * 32 + ks * 8, bdesc, idesc_pv, (i > 0 || ks > 0) ? 1u : 0u);
        }
        umma_commit(p_free + j);
        umma_commit(kv_empty + st);
        return true;
      };
      bool ok = mbar_wait(q_full, 0, wc);
      for (int i = 0; ok && i < min(2, ntiles); ++i) ok = issue_s(i);
      for (int i = 0; ok && i < ntiles; ++i) {
        if (i + 2 < ntiles && !issue_s(i + 2)) { ok = false; break; }
        if (!issue_pv(i)) { ok = false; break; }
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
    const int tid = threadIdx.x - 64;
    // bound of the key norms over this split
    float km = 0.f;
    const float* kn = p.knorm + static_cast<size_t>(bh) * p.n_groups32;
    const int g_end = min(t1 * (kEncTile / kNormGroup), p.n_groups32);
    for (int gi = t0 * (kEncTile / kNormGroup) + tid; gi < g_end; gi += 128) km = fmaxf(km, kn[gi]);
    km = warp_max(km);
    if (lane == 0) red[wq] = km;
    named_bar_sync(1, 128);
    km = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
    float qn = 0.f;
    if (row_ok) {
      const uint4* qrow = reinterpret_cast<const uint4*>(p.q + (static_cast<size_t>(g) * p.M + m) * D);
#pragma unroll
      for (int u = 0; u < D / 8; ++u) {
        const uint4 v = qrow[u];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const float a = bf16_lo(w[t]), bb = bf16_hi(w[t]);
          qn = fmaf(a, a, fmaf(bb, bb, qn));
        }
      }
      qn = sqrtf(qn);
    }
    const float c = p.c;
    const float U = c * qn * km;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    bool ok = true;
    for (int i = 0; i < ntiles; ++i) {
      const int j = i & 1;
      if (!mbar_wait_warp(s_full + j, (i >> 1) & 1, wc)) { ok = false; break; }
      tc_fence_after();
      uint32_t sa[32], sb[32], pk[32];
      if (warp_live) {
        tmem_ld32(lane_base + Cfg::COL_S + j * 64, sa);
        tmem_ld32(lane_base + Cfg::COL_S + j * 64 + 32, sb);
        tmem_wait_ld();
      }
      tc_fence_before();
      mbar_arrive(s_free + j);  // the tensor pipe may now overwrite S[j]
      if (warp_live) {
        const int valid = L - (t0 + i) * kEncTile;
        if (valid >= kEncTile) {
          exp2_chunk64<FLARE_ENC_POLY_PAIRS>(sa, sb, c, U, pk);
        } else {  // last, partial tile of the valid range: padded tokens get weight 0
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const float e0 = (2 * k < valid) ? ex2_mufu(fmaf(__uint_as_float(sa[2 * k]), c, -U)) : 0.f;
            const float e1 = (2 * k + 1 < valid) ? ex2_mufu(fmaf(__uint_as_float(sa[2 * k + 1]), c, -U)) : 0.f;
            const float e2 = (32 + 2 * k < valid) ? ex2_mufu(fmaf(__uint_as_float(sb[2 * k]), c, -U)) : 0.f;
            const float e3 =
                (33 + 2 * k < valid) ? ex2_mufu(fmaf(__uint_as_float(sb[2 * k + 1]), c, -U)) : 0.f;
            pk[k] = pack_bf16x2(e0, e1);
            pk[16 + k] = pack_bf16x2(e2, e3);
          }
        }
      }
      // P[j] was last read by the value MMA of tile i-2
      if (i >= 2 && !mbar_wait_warp(p_free + j, ((i >> 1) - 1) & 1, wc)) { ok = false; break; }
      tc_fence_after();
      if (warp_live) {
        tmem_st32(lane_base + Cfg::COL_P + j * 32, pk);
        tmem_wait_st();
      }
      tc_fence_before();
      mbar_arrive(p_full + j);
    }
    if (ok && mbar_wait_warp(o_full, 0, wc)) {
      tc_fence_after();
      if (warp_live) {
        uint32_t o[32];
        tmem_ld32(lane_base + Cfg::COL_O, o);
        float l;
        if constexpr (D == 16) {
          tmem_wait_ld();
          l = __uint_as_float(o[16]);
        } else {
          uint32_t o2[16];
          tmem_ld16(lane_base + Cfg::COL_O + 32, o2);
          tmem_wait_ld();
          l = __uint_as_float(o2[0]);
        }
        if (row_ok) {
          float* dst = part_base + static_cast<size_t>(m) * (D + 2);
          dst[0] = U;
          dst[1] = l;
#pragma unroll
          for (int d = 0; d < D; ++d) dst[2 + d] = __uint_as_float(o[d]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::TMEM_COLS);
  }
}

}  // namespace

size_t encode_smem_bytes(int D) {
  const size_t need = (D == 16 ? EncCfg<16>::BYTES : EncCfg<32>::BYTES) + 1024;
  // Reserve enough shared memory that at most kSlotsPerSM CTAs share an SM:
  // each CTA holds 256 of the 512 TMEM columns.
  return need > 90 * 1024 ? need : 90 * 1024;
}

cudaError_t launch_encode(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                          const EncodeParams& p, cudaStream_t s) {
  const size_t smem = encode_smem_bytes(p.D);
  const dim3 grid(static_cast<unsigned>(p.B * p.H * p.n_lblocks * p.n_splits));
  if (p.D == 16) {
    cudaError_t e = cudaFuncSetAttribute(encode_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    encode_kernel<16><<<grid, 192, smem, s>>>(tm_q, tm_k, tm_v, p);
  } else {
    cudaError_t e = cudaFuncSetAttribute(encode_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    encode_kernel<32><<<grid, 192, smem, s>>>(tm_q, tm_k, tm_v, p);
  }
  return cudaGetLastError();
}

}  // namespace flare
