// Split-N encoder SDPA on tcgen05 (FLARE++ paper, arXiv 2608.11519, section
// "Method": the FLARE encoder Z_h = softmax_n(Q_h K_h^T / sqrt(D)) V_h of
// eq. 5, which is also the query synthesis of eq. 8 and the encode of eq. 10).
//
// One CTA owns (b, h, a block of 128 latents, a contiguous range of token
// tiles of T tokens, T = enc_tile(D)).  Per tile i:
//   S_i = Q_blk K_i^T             UMMA M=128 (latents) x N=T (tokens), fp32 in TMEM
//   P_i = 2^(S_i * c - U_m)       softmax threads, one latent row per thread
//   O  += P_i [V_i | 1]           UMMA with A = P_i read from TMEM; the ones block
//                                 makes column D of O the running row sum
// The shift U_m = c * |q_m| * max_{n in split} |k_n| is an upper bound of the
// row's scaled scores (Cauchy-Schwarz), fixed for the whole split, so no
// running maximum and no rescaling of O is needed.  The split writes
// (U_m, sum_m, O_m) and the merge kernel combines splits with the exact
// log-sum-exp rule of section "Multi-GPU context parallelism" (eq. 14).
//
// TMEM holds NB score buffers (enc_bufs: two at D = 16, three at D = 32);
// tile i uses buffer i % NB, and the softmax threads write P_i (bf16 pairs)
// over the first T/2 columns of S_i once they hold S_i in registers.
// S_{i+NB} reuses the buffer after the value MMA of tile i has completed.
// The MMA thread issues S_{i+2} right after P_i V_i: with two buffers it
// waits for that value MMA first; with three, S_{i+2}'s buffer last held
// P_{i-1}, whose value MMA finished a tile earlier.  Either way the softmax
// threads find S_{i+1} ready when they finish tile i.  They wait on a single
// barrier per tile (S_i ready); their only other barrier operation is the
// arrive that hands P_i to the MMA thread.  Every barrier that is reused
// across tiles exists once per buffer, so no party can run a full phase
// ahead of the party that waits on it.
//
// Warp roles (5 warps): warp 0 lane 0 is the MMA thread, issuing in program
// order S_0, S_1, P_0 V_0, S_2, P_1 V_1, S_3, ...  Warps 1..4 are the softmax
// warps (thread <-> TMEM lane <-> latent row).  They also refill the K/V
// ring: S_i was issued after P_{i-2} V_{i-2}, so once S_i is complete the
// ring stage of tile i-2 is free, and one softmax warp, in rotation, loads
// tile i-2+NST into it.  A CTA needs 128 TMEM columns for D = 16 (two
// 48-token score buffers and O), so four CTAs (four softmax warps per SM
// sub-partition) share an SM.
#include <type_traits>

#include "ptx.cuh"

namespace flare {
namespace {

template <int D>
struct EncCfg {
  static constexpr int T = enc_tile(D);                // tokens per tile
  static constexpr int ROWB = D * 2;                   // bytes of one K/V/Q row
  static constexpr int TILE_B = T * ROWB;              // bytes of one K or V tile
  static constexpr int Q_B = kLatBlock * ROWB;
  static constexpr int NST = 8;                        // K/V ring stages
  static constexpr uint32_t LAYOUT = (D == 16) ? LAYOUT_SW32 : LAYOUT_SW64;
  static constexpr uint32_t SBO = 8 * ROWB;            // stride of 8-row core-matrix groups
  static constexpr int NO = D + 16;                    // O columns: D values + 16 copies of the sum
  static constexpr int NB = enc_bufs(D);               // score buffers
  // TMEM columns: score buffers at 0, T, 2T (each later holds its P), O at 3T
  static constexpr uint32_t COL_O = NB * T;
  static constexpr uint32_t TMEM_COLS = (COL_O + NO <= 128) ? 128 : 256;
  // Each V stage is followed by its own block of ones, so that [V | 1] has
  // the same leading byte offset (TILE_B) in every stage.
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_B;
  static constexpr int OFF_V = OFF_K + NST * TILE_B;   // NST x [V tile | ones]
  static constexpr int OFF_BAR = OFF_V + NST * 2 * TILE_B;
  static constexpr int OFF_MISC = OFF_BAR + 8 * (2 + NST + 3 * NB);
  static constexpr int BYTES = OFF_MISC + 64 + NST * 4;
  static constexpr int THREADS = 160;
  static constexpr int CTAS_PER_SM = enc_ctas_per_sm(D);
  static_assert(TMEM_COLS <= 512 / CTAS_PER_SM, "TMEM columns of the co-resident CTAs exceed 512");
  static_assert(COL_O + NO <= TMEM_COLS, "score buffers and O exceed the allocation");
  static_assert(T % 16 == 0 && TILE_B % 256 == 0, "tile must hold whole swizzle atoms");
};

template <int D>
__global__ void __launch_bounds__(EncCfg<D>::THREADS, EncCfg<D>::CTAS_PER_SM)
    encode_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const EncodeParams p) {
  using Cfg = EncCfg<D>;
  constexpr int NST = Cfg::NST, T = Cfg::T, NB = Cfg::NB;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sq = sm + Cfg::OFF_Q;
  uint8_t* sk = sm + Cfg::OFF_K;
  uint8_t* sv = sm + Cfg::OFF_V;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Cfg::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;            // [NST] K/V tile landed
  uint64_t* s_full = bars + 1 + NST;       // [NB] score buffer computed
  uint64_t* pv_done = s_full + NB;         // [NB] value MMA done reading the buffer's P
  uint64_t* p_full = s_full + 2 * NB;      // [NB] P stored by every softmax warp (one arrive per warp)
  uint64_t* o_full = s_full + 3 * NB;      // every MMA of the CTA done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + Cfg::OFF_MISC);
  int* abort_flag = reinterpret_cast<int*>(sm + Cfg::OFF_MISC + 4);
  float* red = reinterpret_cast<float*>(sm + Cfg::OFF_MISC + 16);
  volatile int* last_load = reinterpret_cast<volatile int*>(sm + Cfg::OFF_MISC + 64);  // per stage

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int LB = p.n_lblocks, S = p.n_splits;
  const int lb = blockIdx.x % LB;
  const int s = (blockIdx.x / LB) % S;
  const int bh = blockIdx.x / (LB * S);
  const int b = bh / p.H, h = bh % p.H;
  bool bad_len = false;
  const int L = shard_valid_len(p.lengths, b, p.N, p.tok_offset, p.n_global, &bad_len);
  if (bad_len && threadIdx.x == 0) atomicOr(p.err, FLARE_DEV_BAD_LENGTH);
  const int ntiles_valid = (L + T - 1) / T;
  const int t0 = s * p.tiles_per_split;
  const int t1 = min(t0 + p.tiles_per_split, ntiles_valid);
  const int ntiles = max(0, t1 - t0);
  const int g = p.q_per_batch ? bh : h;
  float* part_base = p.part + static_cast<size_t>(bh * S + s) * p.M * (D + 2);
  pdl_launch_dependents();

  if (ntiles == 0) {  // empty split: contributes nothing to the merge
    pdl_wait();
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
      last_load[i] = -1;
    }
    for (int i = 0; i < NB; ++i) {
      mbar_init(s_full + i, 1);
      mbar_init(pv_done + i, 1);
      mbar_init(p_full + i, 4);
    }
    mbar_init(o_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  for (int i = threadIdx.x; i < NST * Cfg::TILE_B / 4; i += blockDim.x) {
    const int st = i / (Cfg::TILE_B / 4), w = i % (Cfg::TILE_B / 4);
    reinterpret_cast<uint32_t*>(sv + (2 * st + 1) * Cfg::TILE_B)[w] = 0x3F803F80u;  // bf16 1.0 pairs
  }
  fence_proxy_async_smem();
  if (warp == 0) {
    tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // set-up done: from here on global memory that the previous kernel writes
  pdl_wait();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx wc{p.err, abort_flag, p.timeout_ns};
  // K and V of tile n into ring stage n % NST (one thread)
  auto load_tile = [&](int n) {
    const int st = n % NST;
    mbar_arrive_expect_tx(kv_full + st, 2 * Cfg::TILE_B);
    const int tok = (t0 + n) * T;
    tma_load_3d(sk + st * Cfg::TILE_B, &tm_k, kv_full + st, 0, tok, bh);
    tma_load_3d(sv + st * 2 * Cfg::TILE_B, &tm_v, kv_full + st, 0, tok, bh);
    last_load[st] = n;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ MMA thread
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      mbar_arrive_expect_tx(q_full, p.q_rows * Cfg::ROWB);
      tma_load_3d(sq, &tm_q, q_full, 0, lb * kLatBlock, g);
      for (int n = 0; n < min(NST, ntiles); ++n) load_tile(n);
      const uint32_t idesc_s = idesc_bf16_f32(128, T, false, false);
      const uint32_t idesc_pv = idesc_bf16_f32(128, Cfg::NO, false, true);
      // descriptors of stage 0; a stage's descriptor adds its byte offset >> 4
      const uint64_t q_desc = umma_desc(smem_u32(sq), 16, Cfg::SBO, Cfg::LAYOUT);
      const uint64_t k_desc = umma_desc(smem_u32(sk), 16, Cfg::SBO, Cfg::LAYOUT);
      const uint64_t v_desc = umma_desc(smem_u32(sv), Cfg::TILE_B, Cfg::SBO, Cfg::LAYOUT);
      // S_i into buffer i % NB, once tile i has landed and P_{i-NB} has been consumed
      auto issue_s = [&](int i) -> bool {
        const int st = i % NST, buf = i % NB;
        if (!mbar_wait_mma(kv_full + st, (i / NST) & 1, wc)) return false;
        if (i >= NB && !mbar_wait_mma(pv_done + buf, ((i - NB) / NB) & 1, wc)) return false;
        tc_fence_after();
        const uint64_t kd = k_desc + static_cast<uint64_t>((st * Cfg::TILE_B) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          umma_ss(tmem + buf * T, q_desc + 2 * kk, kd + 2 * kk, idesc_s, kk > 0 ? 1u : 0u);
        umma_commit(s_full + buf);
        return true;
      };
      // O += P_i [V_i | 1] once every softmax warp has stored P_i
      auto issue_pv = [&](int i) -> bool {
        const int buf = i % NB;
        if (!mbar_wait_mma(p_full + buf, (i / NB) & 1, wc)) return false;
        tc_fence_after();
        const uint64_t vd = v_desc + static_cast<uint64_t>(((i % NST) * 2 * Cfg::TILE_B) >> 4);
#pragma unroll
        for (int ks = 0; ks < T / 16; ++ks)
          umma_ts(tmem + Cfg::COL_O, tmem + buf * T + ks * 8, vd + static_cast<uint64_t>((ks * 16 * Cfg::ROWB) >> 4),
                  idesc_pv, (i > 0 || ks > 0) ? 1u : 0u);
        umma_commit(pv_done + buf);
        return true;
      };
      bool ok = mbar_wait_mma(q_full, 0, wc) && issue_s(0);
      if (ok && ntiles > 1) ok = issue_s(1);
      for (int i = 0; ok && i < ntiles; ++i) {
        ok = issue_pv(i);
        if (ok && i + 2 < ntiles) ok = issue_s(i + 2);
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
    const int tid = threadIdx.x - 32;
    // bound of the key norms over this split (the 32-token groups that
    // overlap its token range)
    float km = 0.f;
    const float* kn = p.knorm + static_cast<size_t>(bh) * p.n_groups32;
    const int g_beg = (t0 * T) / kNormGroup;
    const int g_end = min((t1 * T + kNormGroup - 1) / kNormGroup, p.n_groups32);
    for (int gi = g_beg + tid; gi < g_end; gi += 128) km = fmaxf(km, kn[gi]);
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
    // the tile loop, with NP polynomial exp2 pairs out of every 32
    auto run_tiles = [&](auto np_tag) -> bool {
      constexpr int NP = decltype(np_tag)::value;
      for (int i = 0, buf = 0, use = 0; i < ntiles; ++i) {
        if (!mbar_wait_warp(s_full + buf, use & 1, wc)) return false;
        tc_fence_after();
        const int valid = L - (t0 + i) * T;
        if (warp_live && FLARE_ENC_SPLIT_LD && valid >= T) {
          // first 16 columns, then the rest while the first are exponentiated
          constexpr int R = T - 16;
          uint32_t s0[16], s1[R], pk[T / 2];
          tmem_ld16(lane_base + buf * T, s0);
          tmem_wait_ld();
          tmem_ld_cols<R>(lane_base + buf * T + 16, s1);
          exp2_row<16, NP>(s0, c, U, *reinterpret_cast<uint32_t(*)[8]>(&pk[0]));
          tmem_wait_ld();
          exp2_row<R, NP, 8>(s1, c, U, *reinterpret_cast<uint32_t(*)[R / 2]>(&pk[8]));
          tmem_st_cols<T / 2>(lane_base + buf * T, pk);  // P_i over the first T/2 columns of S_i
          tmem_wait_st();
        } else if (warp_live) {
          uint32_t sc[T], pk[T / 2];
          tmem_ld_cols<T>(lane_base + buf * T, sc);
          tmem_wait_ld();
          if (valid >= T) {
            exp2_row<T, NP>(sc, c, U, pk);
          } else {  // last, partial tile of the valid range: padded tokens get weight 0
#pragma unroll
            for (int k = 0; k < T / 2; ++k) {
              const float e0 = (2 * k < valid) ? ex2_mufu(fmaf(__uint_as_float(sc[2 * k]), c, -U)) : 0.f;
              const float e1 = (2 * k + 1 < valid) ? ex2_mufu(fmaf(__uint_as_float(sc[2 * k + 1]), c, -U)) : 0.f;
              pk[k] = pack_bf16x2(e0, e1);
            }
          }
          tmem_st_cols<T / 2>(lane_base + buf * T, pk);  // P_i over the first T/2 columns of S_i
          tmem_wait_st();
        }
        tc_fence_before();
        mbar_arrive_warp(p_full + buf);
        // S_i complete implies P_{i-2} V_{i-2} complete: its ring stage is free
        if (i >= 2 && i - 2 + NST < ntiles && wq == (i & 3) && lane == 0) load_tile(i - 2 + NST);
        __syncwarp();
        if (++buf == NB) {
          buf = 0;
          ++use;
        }
      }
      return true;
    };
    const bool ok = run_tiles(std::integral_constant<int, FLARE_ENC_POLY_PAIRS>{});
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
    if (lane == 0) {  // copies still in flight (only after an abort) must land before exit
      for (int st = 0; st < NST; ++st)
        if (last_load[st] >= 0) mbar_wait_drain(kv_full + st, (last_load[st] / NST) & 1, p.timeout_ns);
      mbar_wait_drain(q_full, 0, p.timeout_ns);
    }
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::TMEM_COLS);
  }
}

}  // namespace

size_t encode_smem_bytes(int D) {
  const size_t need = (D == 16 ? EncCfg<16>::BYTES : EncCfg<32>::BYTES) + 1024;
  // Reserve enough shared memory that at most enc_ctas_per_sm(D) CTAs share
  // an SM (228 KB each, 1 KB of it reserved per CTA), so that every resident
  // CTA finds its TMEM columns free.
  const size_t floor = (228 * 1024) / (enc_ctas_per_sm(D) + 1) + 1024;
  return need > floor ? need : floor;
}

cudaError_t launch_encode(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                          const EncodeParams& p, cudaStream_t s, bool pdl) {
  const size_t smem = encode_smem_bytes(p.D);
  const dim3 grid(static_cast<unsigned>(p.B * p.H * p.n_lblocks * p.n_splits));
  auto go = [&](auto kern, int threads) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    LaunchCfg lc(grid, dim3(threads), smem, s, pdl);
    return cudaLaunchKernelEx(&lc.cfg, kern, tm_q, tm_k, tm_v, p);
  };
  return p.D == 16 ? go(encode_kernel<16>, EncCfg<16>::THREADS) : go(encode_kernel<32>, EncCfg<32>::THREADS);
}

}  // namespace flare
