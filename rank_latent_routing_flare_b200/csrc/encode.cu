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
// Warp roles (5 warps): warp 0 lane 0 is the control thread: it keeps the
// K/V ring full (TMA) and issues the MMAs in program order, blocking on
// exactly the next event (S(i+1) once every softmax warp has loaded S(i);
// P(i) [V(i) | 1] once every softmax warp has stored P(i)).  Warps 1..4 are
// the softmax warps (thread <-> TMEM lane <-> latent row).  A CTA needs 128
// TMEM columns for D = 16: three CTAs (three softmax warps per SM
// sub-partition) share an SM.
#include "ptx.cuh"

namespace flare {
namespace {

template <int D>
struct EncCfg {
  static constexpr int T = kEncTile;                   // tokens per tile (64)
  static constexpr int ROWB = D * 2;                   // bytes of one K/V/Q row
  static constexpr int TILE_B = T * ROWB;              // bytes of one K or V tile
  static constexpr int Q_B = kLatBlock * ROWB;
  static constexpr int NST = 8;                        // K/V ring stages
  static constexpr uint32_t LAYOUT = (D == 16) ? LAYOUT_SW32 : LAYOUT_SW64;
  static constexpr uint32_t SBO = 8 * ROWB;            // stride of 8-row core-matrix groups
  static constexpr int NO = D + 16;                    // O columns: D values + 16 copies of the sum
  // TMEM columns: S at 0 (fp32 scores), P at T (bf16 pairs), O at 3T/2
  static constexpr uint32_t COL_S = 0, COL_P = T, COL_O = T + T / 2;
  static constexpr uint32_t TMEM_COLS = (COL_O + NO <= 128) ? 128 : 256;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_B;
  static constexpr int OFF_V = OFF_K + NST * TILE_B;
  static constexpr int OFF_ONES = OFF_V + NST * TILE_B;
  static constexpr int OFF_BAR = OFF_ONES + TILE_B;
  static constexpr int OFF_MISC = OFF_BAR + 8 * 32;
  static constexpr int BYTES = OFF_MISC + 64;
  static constexpr int THREADS = 160;
  static constexpr int CTAS_PER_SM = enc_ctas_per_sm(D);
};

template <int D>
__global__ void __launch_bounds__(EncCfg<D>::THREADS, EncCfg<D>::CTAS_PER_SM)
    encode_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const EncodeParams p) {
  using Cfg = EncCfg<D>;
  constexpr int NST = Cfg::NST, T = Cfg::T;
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
  uint64_t* s_full = bars + 1 + 2 * NST;  // S computed
  uint64_t* s_free = s_full + 1;           // S loaded by every softmax warp (one arrive per warp)
  uint64_t* p_full = s_full + 2;           // P stored by every softmax warp (one arrive per warp)
  uint64_t* p_free = s_full + 3;           // P consumed by the value MMA
  uint64_t* o_full = s_full + 4;           // every MMA of the CTA done
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
  const int ntiles_valid = (L + T - 1) / T;
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
    mbar_init(s_full, 1);
    mbar_init(s_free, 4);
    mbar_init(p_full, 4);
    mbar_init(p_free, 1);
    mbar_init(o_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  for (int i = threadIdx.x; i < Cfg::TILE_B / 4; i += blockDim.x)
    reinterpret_cast<uint32_t*>(sones)[i] = 0x3F803F80u;  // bf16 1.0 pairs
  fence_proxy_async_smem();
  if (warp == 0) {
    tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx wc{p.err, abort_flag, p.timeout_ns};

  if (warp == 0) {
    // ------------------------------------------------------------ control thread
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      mbar_arrive_expect_tx(q_full, p.q_rows * Cfg::ROWB);
      tma_load_3d(sq, &tm_q, q_full, 0, lb * kLatBlock, g);
      const uint32_t idesc_s = idesc_bf16_f32(128, T, false, false);
      const uint32_t idesc_pv = idesc_bf16_f32(128, Cfg::NO, false, true);
      const uint32_t sq_a = smem_u32(sq), ones_a = smem_u32(sones);
      int n_load = 0;
      auto load = [&]() {
        const int st = n_load % NST;
        mbar_arrive_expect_tx(kv_full + st, 2 * Cfg::TILE_B);
        const int tok = (t0 + n_load) * T;
        tma_load_3d(sk + st * Cfg::TILE_B, &tm_k, kv_full + st, 0, tok, bh);
        tma_load_3d(sv + st * Cfg::TILE_B, &tm_v, kv_full + st, 0, tok, bh);
        ++n_load;
      };
      // refill every ring stage whose previous tile's value MMA has completed
      auto refill = [&]() {
        while (n_load < ntiles && mbar_test(kv_empty + n_load % NST, ((n_load / NST) & 1) ^ 1)) load();
      };
      auto issue_s = [&](int i) -> bool {
        while (n_load <= i) {  // tile i not requested yet: wait for its stage
          if (!mbar_wait(kv_empty + n_load % NST, ((n_load / NST) & 1) ^ 1, wc)) return false;
          load();
        }
        if (!mbar_wait(kv_full + i % NST, (i / NST) & 1, wc)) return false;
        tc_fence_after();
        const uint32_t k_a = smem_u32(sk + (i % NST) * Cfg::TILE_B);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          umma_ss(tmem + Cfg::COL_S, umma_desc(sq_a + kk * 32, 16, Cfg::SBO, Cfg::LAYOUT),
                  umma_desc(k_a + kk * 32, 16, Cfg::SBO, Cfg::LAYOUT), idesc_s, kk > 0 ? 1u : 0u);
        umma_commit(s_full);
        return true;
      };
      auto issue_pv = [&](int i) -> bool {
        if (!mbar_wait(p_full, i & 1, wc)) return false;
        tc_fence_after();
        const int st = i % NST;
        const uint32_t v_a = smem_u32(sv + st * Cfg::TILE_B);
        const uint32_t lbo = ones_a - v_a;  // [V | 1] : second N-atom = ones block
#pragma unroll
        for (int ks = 0; ks < T / 16; ++ks) {
          const uint64_t bdesc = umma_desc(v_a + ks * 16 * Cfg::ROWB, lbo, Cfg::SBO, Cfg::LAYOUT);
          umma_ts(tmem + Cfg::COL_O, tmem + Cfg::COL_P + ks * 8, bdesc, idesc_pv, (i > 0 || ks > 0) ? 1u : 0u);
        }
        umma_commit(p_free);
        umma_commit(kv_empty + st);
        return true;
      };
      refill();
      bool ok = mbar_wait(q_full, 0, wc) && issue_s(0);
      for (int i = 1; ok && i < ntiles; ++i) {
        ok = mbar_wait(s_free, (i - 1) & 1, wc) && issue_s(i);  // S(i-1) loaded -> S(i)
        if (ok) ok = issue_pv(i - 1);                             // P(i-1) stored -> P(i-1) V(i-1)
        if (ok) refill();
      }
      if (ok) issue_pv(ntiles - 1);
      umma_commit(o_full);  // completes once every MMA issued above is done
      mbar_wait_drain(o_full, 0, p.timeout_ns);
      for (int i = max(0, n_load - NST); i < n_load; ++i)  // copies in flight must land
        mbar_wait_drain(kv_full + (i % NST), (i / NST) & 1, p.timeout_ns);
      mbar_wait_drain(q_full, 0, p.timeout_ns);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int wq = warp & 3;                  // TMEM lane quarter of this warp
    const int r = wq * 32 + lane;             // latent row within the block
    const int m = lb * kLatBlock + r;
    const bool row_ok = m < p.M;
    const bool warp_live = lb * kLatBlock + wq * 32 < p.M;
    const int tid = threadIdx.x - 32;
    // bound of the key norms over this split
    float km = 0.f;
    const float* kn = p.knorm + static_cast<size_t>(bh) * p.n_groups32;
    const int g_end = min(t1 * (T / kNormGroup), p.n_groups32);
    for (int gi = t0 * (T / kNormGroup) + tid; gi < g_end; gi += 128) km = fmaxf(km, kn[gi]);
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
      if (!mbar_wait_warp(s_full, i & 1, wc)) { ok = false; break; }
      tc_fence_after();
      uint32_t sa[32], sb[32], pk[32];
      if (warp_live) {
        tmem_ld32(lane_base + Cfg::COL_S, sa);
        tmem_ld32(lane_base + Cfg::COL_S + 32, sb);
        tmem_wait_ld();
      }
      tc_fence_before();
      mbar_arrive_warp(s_free);  // the tensor pipe may now write S(i+1)
      if (warp_live) {
        const int valid = L - (t0 + i) * T;
        if (valid >= T) {
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
      // P was last read by the value MMA of tile i-1
      if (i >= 1 && !mbar_wait_warp(p_free, (i - 1) & 1, wc)) { ok = false; break; }
      tc_fence_after();
      if (warp_live) {
        tmem_st32(lane_base + Cfg::COL_P, pk);
        tmem_wait_st();
      }
      tc_fence_before();
      mbar_arrive_warp(p_full);
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
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::TMEM_COLS);
  }
}

}  // namespace

size_t encode_smem_bytes(int D) {
  const size_t need = (D == 16 ? EncCfg<16>::BYTES : EncCfg<32>::BYTES) + 1024;
  // Reserve enough shared memory that at most enc_ctas_per_sm(D) CTAs share
  // an SM, so that every resident CTA finds its TMEM columns free.
  const size_t floor = enc_ctas_per_sm(D) >= 3 ? 70 * 1024 : 100 * 1024;
  return need > floor ? need : floor;
}

cudaError_t launch_encode(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                          const EncodeParams& p, cudaStream_t s) {
  const size_t smem = encode_smem_bytes(p.D);
  const dim3 grid(static_cast<unsigned>(p.B * p.H * p.n_lblocks * p.n_splits));
  if (p.D == 16) {
    cudaError_t e = cudaFuncSetAttribute(encode_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    encode_kernel<16><<<grid, EncCfg<16>::THREADS, smem, s>>>(tm_q, tm_k, tm_v, p);
  } else {
    cudaError_t e = cudaFuncSetAttribute(encode_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    encode_kernel<32><<<grid, EncCfg<32>::THREADS, smem, s>>>(tm_q, tm_k, tm_v, p);
  }
  return cudaGetLastError();
}

}  // namespace flare
