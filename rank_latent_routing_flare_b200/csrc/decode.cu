// Decoder SDPA on tcgen05 (FLARE++ paper, arXiv 2608.11519, section "Method":
// the FLARE decoder Y_h = softmax_m(K_h Q_h^T / sqrt(D)) Z_h of eq. 6, used
// with Q_h(X) in eq. 11).
//
// One CTA owns one head (b, h) and a contiguous range of 128-token tiles.  The
// head's queries Q (M x D) and latent values Z (M x D) stay resident in shared
// memory; key tiles stream through a TMA ring.  Per tile and per 64-latent
// chunk c:
//   S = K_tile Q_c^T               UMMA M=128 (tokens) x N=64 (latents), fp32 TMEM
//   P = 2^(S * c - nu_n)           softmax threads, one token row per thread
//   Y += P [Z_c | 1]               UMMA with A = P read from TMEM; column D of Y
//                                  accumulates the row sum
// nu_n = c * |k_n| * max_m |q_m| bounds the token's scaled scores from above
// (Cauchy-Schwarz), so the latent chunks need no running maximum.  A token
// whose sum underflows (only possible when the bound is very loose) is
// recomputed exactly by its own thread from global memory.
//
// Warp roles (5 warps): warp 0 lane 0 is the control thread: it loads Q and
// Z, keeps the key-tile ring full (TMA) and issues the MMAs in program order,
// blocking on exactly the next event.  Warps 1..4 are the softmax warps
// (thread <-> TMEM lane <-> token).  A CTA needs 128 TMEM columns for D = 16,
// so three CTAs share an SM.
#include "ptx.cuh"

namespace flare {
namespace {

template <int D>
struct DecCfg {
  static constexpr int ROWB = D * 2;
  static constexpr int KT_B = kDecTile * ROWB;          // one key tile
  static constexpr int CH_B = kDecChunk * ROWB;         // one 64-latent chunk of Q or Z
  static constexpr int MAXCH = 512 / kDecChunk;         // M <= 512
  static constexpr int NST = 4;
  static constexpr uint32_t LAYOUT = (D == 16) ? LAYOUT_SW32 : LAYOUT_SW64;
  static constexpr uint32_t SBO = 8 * ROWB;
  static constexpr int NY = D + 16;                     // Y columns: D values + sums
  static constexpr int OFF_Q = 0;                       // MAXCH * CH_B
  static constexpr int OFF_Z = OFF_Q + MAXCH * CH_B;
  static constexpr int OFF_ONES = OFF_Z + MAXCH * CH_B; // CH_B
  static constexpr int OFF_K = OFF_ONES + CH_B;         // NST * KT_B
  static constexpr int OFF_BAR = OFF_K + NST * KT_B;
  static constexpr int OFF_MISC = OFF_BAR + 8 * 32;
  static constexpr int BYTES = OFF_MISC + 64;
  // TMEM columns: S at 0 (fp32 scores of one 64-latent chunk), P at 64 (bf16
  // pairs), Y at 96 (D values + the row-sum block)
  static constexpr uint32_t COL_S = 0, COL_P = 64, COL_Y = 96;
  static constexpr uint32_t TMEM_COLS = (COL_Y + NY <= 128) ? 128 : 256;
  static constexpr int THREADS = 160;
  static constexpr int CTAS_PER_SM = dec_ctas_per_sm(D);
};

__device__ __forceinline__ float bf16_row_norm2(const uint4* row, int n16) {
  float s = 0.f;
  for (int u = 0; u < n16; ++u) {
    const uint4 v = row[u];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const float a = bf16_lo(w[t]), b = bf16_hi(w[t]);
      s = fmaf(a, a, fmaf(b, b, s));
    }
  }
  return s;
}

// Exact two-pass softmax over the M latents for one token, written straight
// to its output row: the fallback for tokens whose fast-path row sum
// underflowed (only possible when the norm bound is very loose).  fp32 from
// global memory; one thread per listed token.
template <int D>
__global__ void __launch_bounds__(128) decode_fallback_kernel(const DecodeParams p) {
  const uint32_t count = *p.fb_count;
  for (uint32_t e = blockIdx.x * blockDim.x + threadIdx.x; e < count; e += gridDim.x * blockDim.x) {
    const uint64_t tok = p.fb_list[e];
    const int bh = static_cast<int>(tok / static_cast<uint64_t>(p.N));
    const int n = static_cast<int>(tok % static_cast<uint64_t>(p.N));
    const int g = p.q_per_batch ? bh : bh % p.H;
    const uint16_t* krow = p.k + (static_cast<size_t>(bh) * p.N + n) * D;
    const uint16_t* qg = p.q + static_cast<size_t>(g) * p.M * D;
    const uint16_t* zh = p.z + static_cast<size_t>(bh) * p.M * D;
    float k[D], y[D];
#pragma unroll
    for (int d = 0; d < D; ++d) k[d] = __uint_as_float(static_cast<uint32_t>(krow[d]) << 16);
    float mx = -INFINITY;
    for (int m = 0; m < p.M; ++m) {
      float s = 0.f;
#pragma unroll
      for (int d = 0; d < D; ++d) s = fmaf(k[d], __uint_as_float(static_cast<uint32_t>(qg[m * D + d]) << 16), s);
      mx = fmaxf(mx, s * p.c);
    }
    float den = 0.f;
#pragma unroll
    for (int d = 0; d < D; ++d) y[d] = 0.f;
    for (int m = 0; m < p.M; ++m) {
      float s = 0.f;
#pragma unroll
      for (int d = 0; d < D; ++d) s = fmaf(k[d], __uint_as_float(static_cast<uint32_t>(qg[m * D + d]) << 16), s);
      const float w = exp2f(s * p.c - mx);
      den += w;
#pragma unroll
      for (int d = 0; d < D; ++d) y[d] = fmaf(w, __uint_as_float(static_cast<uint32_t>(zh[m * D + d]) << 16), y[d]);
    }
    const float inv = 1.f / den;
    uint4* dst = reinterpret_cast<uint4*>(p.y + (static_cast<size_t>(bh) * p.N + n) * D);
#pragma unroll
    for (int u = 0; u < D / 8; ++u)
      dst[u] = make_uint4(pack_bf16x2(y[8 * u + 0] * inv, y[8 * u + 1] * inv),
                          pack_bf16x2(y[8 * u + 2] * inv, y[8 * u + 3] * inv),
                          pack_bf16x2(y[8 * u + 4] * inv, y[8 * u + 5] * inv),
                          pack_bf16x2(y[8 * u + 6] * inv, y[8 * u + 7] * inv));
  }
}

template <int D>
__global__ void __launch_bounds__(DecCfg<D>::THREADS, DecCfg<D>::CTAS_PER_SM)
    decode_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_z,
                  const __grid_constant__ CUtensorMap tm_k, const DecodeParams p) {
  using Cfg = DecCfg<D>;
  constexpr int NST = Cfg::NST;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sq = sm + Cfg::OFF_Q;
  uint8_t* sz = sm + Cfg::OFF_Z;
  uint8_t* sones = sm + Cfg::OFF_ONES;
  uint8_t* sk = sm + Cfg::OFF_K;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Cfg::OFF_BAR);
  uint64_t* qz_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = bars + 1 + NST;
  uint64_t* s_full = bars + 1 + 2 * NST;  // S computed
  uint64_t* s_free = s_full + 1;           // S loaded by every softmax warp
  uint64_t* p_full = s_full + 2;           // P stored by every softmax warp
  uint64_t* p_free = s_full + 3;           // P consumed by the value MMA
  uint64_t* y_full = s_full + 4;           // Y of a tile complete
  uint64_t* y_free = s_full + 5;           // Y read by every softmax warp
  uint64_t* mma_done = s_full + 6;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + Cfg::OFF_MISC);
  int* abort_flag = reinterpret_cast<int*>(sm + Cfg::OFF_MISC + 4);
  float* red = reinterpret_cast<float*>(sm + Cfg::OFF_MISC + 16);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.x / p.ctas_per_head;
  const int part = blockIdx.x % p.ctas_per_head;
  const int b = bh / p.H, h = bh % p.H;
  const int g = p.q_per_batch ? bh : h;
  int L = p.N;
  if (p.lengths) {
    int l = p.lengths[b];
    if (l < 1 || l > p.N) {
      if (threadIdx.x == 0) atomicOr(p.err, FLARE_DEV_BAD_LENGTH);
      l = min(max(l, 0), p.N);
    }
    L = l;
  }
  const int tiles_head = (p.N + kDecTile - 1) / kDecTile;
  const int tiles_valid = (L + kDecTile - 1) / kDecTile;
  const int ta = part * p.tiles_per_cta;
  const int tb = min(ta + p.tiles_per_cta, tiles_head);
  const int tc_end = min(tb, tiles_valid);            // tiles [ta, tc_end) are computed
  const int ntiles = max(0, tc_end - ta);
  const int nc = (p.M + kDecChunk - 1) / kDecChunk;   // latent chunks
  uint16_t* yh = p.y + static_cast<size_t>(bh) * p.N * D;

  // tiles entirely past the valid length: zero rows
  {
    const int z0 = max(ta, tiles_valid) * kDecTile;
    const int z1 = min(tb * kDecTile, p.N);
    const uint4 zero = make_uint4(0, 0, 0, 0);
    for (size_t e = static_cast<size_t>(z0) * (D / 8) + threadIdx.x; e < static_cast<size_t>(z1) * (D / 8);
         e += blockDim.x)
      reinterpret_cast<uint4*>(yh)[e] = zero;
  }
  if (ntiles == 0) return;

  if (threadIdx.x == 0) {
    mbar_init(qz_full, 1);
    for (int i = 0; i < NST; ++i) {
      mbar_init(k_full + i, 1);
      mbar_init(k_empty + i, 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, 4);
    mbar_init(p_full, 4);
    mbar_init(p_free, 1);
    mbar_init(y_full, 1);
    mbar_init(y_free, 4);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  for (int i = threadIdx.x; i < Cfg::CH_B / 4; i += blockDim.x)
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
      tma_prefetch_desc(&tm_z);
      tma_prefetch_desc(&tm_k);
      mbar_arrive_expect_tx(qz_full, 2 * nc * p.chunk_rows * Cfg::ROWB);
      for (int c = 0; c < nc; ++c) {
        tma_load_3d(sq + c * Cfg::CH_B, &tm_q, qz_full, 0, c * kDecChunk, g);
        tma_load_3d(sz + c * Cfg::CH_B, &tm_z, qz_full, 0, c * kDecChunk, bh);
      }
      const uint32_t idesc_y = idesc_bf16_f32(128, Cfg::NY, false, true);
      const uint32_t sq_a = smem_u32(sq), sz_a = smem_u32(sz), ones_a = smem_u32(sones);
      auto chunk_n = [&](int cc) { return min(kDecChunk, p.M - cc * kDecChunk); };
      int n_load = 0;
      auto load = [&]() {
        const int st = n_load % NST;
        mbar_arrive_expect_tx(k_full + st, Cfg::KT_B);
        tma_load_3d(sk + st * Cfg::KT_B, &tm_k, k_full + st, 0, (ta + n_load) * kDecTile, bh);
        ++n_load;
      };
      auto refill = [&]() {
        while (n_load < ntiles && mbar_test(k_empty + n_load % NST, ((n_load / NST) & 1) ^ 1)) load();
      };
      auto issue_s = [&](int qq) -> bool {
        const int tile = qq / nc, cc = qq - tile * nc;
        const int st = tile % NST;
        if (cc == 0) {
          while (n_load <= tile) {
            if (!mbar_wait(k_empty + n_load % NST, ((n_load / NST) & 1) ^ 1, wc)) return false;
            load();
          }
          if (!mbar_wait(k_full + st, (tile / NST) & 1, wc)) return false;
        }
        tc_fence_after();
        const uint32_t k_a = smem_u32(sk + st * Cfg::KT_B);
        const uint32_t idesc_s = idesc_bf16_f32(128, chunk_n(cc), false, false);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          umma_ss(tmem + Cfg::COL_S, umma_desc(k_a + kk * 32, 16, Cfg::SBO, Cfg::LAYOUT),
                  umma_desc(sq_a + cc * Cfg::CH_B + kk * 32, 16, Cfg::SBO, Cfg::LAYOUT), idesc_s, kk > 0 ? 1u : 0u);
        umma_commit(s_full);
        return true;
      };
      auto issue_pv = [&](int qq) -> bool {
        const int tile = qq / nc, cc = qq - tile * nc;
        // the first value MMA of a tile overwrites Y: the previous tile's
        // epilogue must have read it
        if (cc == 0 && tile >= 1 && !mbar_wait(y_free, (tile - 1) & 1, wc)) return false;
        if (!mbar_wait(p_full, qq & 1, wc)) return false;
        tc_fence_after();
        const uint32_t z_a = sz_a + cc * Cfg::CH_B;
        const uint32_t lbo = ones_a - z_a;  // [Z_c | 1]: second N-atom = ones block
        const int nks = chunk_n(cc) / 16;
        for (int ks = 0; ks < nks; ++ks) {
          const uint64_t bdesc = umma_desc(z_a + ks * 16 * Cfg::ROWB, lbo, Cfg::SBO, Cfg::LAYOUT);
          umma_ts(tmem + Cfg::COL_Y, tmem + Cfg::COL_P + ks * 8, bdesc, idesc_y, (cc > 0 || ks > 0) ? 1u : 0u);
        }
        umma_commit(p_free);
        if (cc == nc - 1) {
          umma_commit(y_full);
          umma_commit(k_empty + (tile % NST));
        }
        return true;
      };
      const int total = ntiles * nc;
      refill();
      bool ok = mbar_wait(qz_full, 0, wc) && issue_s(0);
      for (int qq = 1; ok && qq < total; ++qq) {
        ok = mbar_wait(s_free, (qq - 1) & 1, wc) && issue_s(qq);  // S(q-1) loaded -> S(q)
        if (ok) ok = issue_pv(qq - 1);                              // P(q-1) stored -> P(q-1) [Z | 1]
        if (ok) refill();
      }
      if (ok) issue_pv(total - 1);
      umma_commit(mma_done);  // every MMA issued above is complete before TMEM is freed
      mbar_wait_drain(mma_done, 0, p.timeout_ns);
      for (int i = max(0, n_load - NST); i < n_load; ++i)
        mbar_wait_drain(k_full + (i % NST), (i / NST) & 1, p.timeout_ns);
      mbar_wait_drain(qz_full, 0, p.timeout_ns);
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int wq = warp & 3;
    const int r = wq * 32 + lane;                     // token row within the tile
    const int tid = threadIdx.x - 32;
    const uint16_t* qg = p.q + static_cast<size_t>(g) * p.M * D;
    // largest query norm of the head
    float qm = 0.f;
    for (int m = tid; m < p.M; m += 128)
      qm = fmaxf(qm, bf16_row_norm2(reinterpret_cast<const uint4*>(qg + static_cast<size_t>(m) * D), D / 8));
    qm = warp_max(qm);
    if (lane == 0) red[wq] = qm;
    named_bar_sync(1, 128);
    qm = sqrtf(fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3])));
    const float c = p.c;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    // Epilogue of tile i: Y = acc / sum, zero rows for padding, bf16 stores.
    // It runs inside chunk 0 of tile i+1, after the P store (the value MMA of
    // the tile's last chunk has completed by then).
    auto epilogue = [&](int i) -> bool {
      if (!mbar_wait_warp(y_full, i & 1, wc)) return false;
      tc_fence_after();
      uint32_t o[32];
      float l;
      float y[D];
      tmem_ld32(lane_base + Cfg::COL_Y, o);
      if constexpr (D == 16) {
        tmem_wait_ld();
        l = __uint_as_float(o[16]);
#pragma unroll
        for (int d = 0; d < 16; ++d) y[d] = __uint_as_float(o[d]);
      } else {
        uint32_t o2[16];
        tmem_ld16(lane_base + Cfg::COL_Y + 32, o2);
        tmem_wait_ld();
        l = __uint_as_float(o2[0]);
#pragma unroll
        for (int d = 0; d < 32; ++d) y[d] = __uint_as_float(o[d]);
      }
      tc_fence_before();
      mbar_arrive_warp(y_free);  // the next tile's first value MMA may overwrite Y
      const int n = (ta + i) * kDecTile + r;
      // lost mass < M * 2^-126 per token; 2^-90 keeps it below 2^-27 relative
      const bool exact = n < L && !(l >= 0x1p-90f);
      if (n < L) {
        const float inv = 1.f / l;
#pragma unroll
        for (int d = 0; d < D; ++d) y[d] *= inv;
      } else {
#pragma unroll
        for (int d = 0; d < D; ++d) y[d] = 0.f;
      }
      if (exact) {  // recomputed exactly by decode_fallback_kernel
        const uint32_t e = atomicAdd(p.fb_count, 1u);
        p.fb_list[e] = static_cast<uint64_t>(bh) * p.N + n;
      } else if (n < p.N) {
        uint4* dst = reinterpret_cast<uint4*>(yh + static_cast<size_t>(n) * D);
#pragma unroll
        for (int u = 0; u < D / 8; ++u)
          dst[u] = make_uint4(pack_bf16x2(y[8 * u + 0], y[8 * u + 1]), pack_bf16x2(y[8 * u + 2], y[8 * u + 3]),
                              pack_bf16x2(y[8 * u + 4], y[8 * u + 5]), pack_bf16x2(y[8 * u + 6], y[8 * u + 7]));
      }
      return true;
    };
    const int total = ntiles * nc;
    bool ok = true;
    float nu = 0.f;
    for (int qq = 0; qq < total; ++qq) {
      const int tile = qq / nc, cc = qq - tile * nc;
      if (!mbar_wait_warp(s_full, qq & 1, wc)) { ok = false; break; }
      tc_fence_after();
      const int cn = min(kDecChunk, p.M - cc * kDecChunk);
      uint32_t sa[32], sb[32], pk[32];
      tmem_ld32(lane_base + Cfg::COL_S, sa);
      if (cn > 32) tmem_ld32(lane_base + Cfg::COL_S + 32, sb);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive_warp(s_free);  // the tensor pipe may now write S(q+1)
      if (cc == 0) {
        // |k_n| from the key tile in shared memory (the swizzle only permutes
        // 16-byte halves inside each row, which a sum of squares ignores);
        // the tile stays resident until the tile's last value MMA completes
        const uint4* krow_s = reinterpret_cast<const uint4*>(sk + (tile % NST) * Cfg::KT_B + r * Cfg::ROWB);
        nu = c * sqrtf(bf16_row_norm2(krow_s, D / 8)) * qm;
      }
      if (cn == kDecChunk) {
        exp2_chunk64<FLARE_DEC_POLY_PAIRS>(sa, sb, c, nu, pk);
      } else if (cn > 32) {  // 48 latents
#pragma unroll
        for (int k = 0; k < 16; ++k)
          pk[k] = pack_bf16x2(ex2_mufu(fmaf(__uint_as_float(sa[2 * k]), c, -nu)),
                              ex2_mufu(fmaf(__uint_as_float(sa[2 * k + 1]), c, -nu)));
#pragma unroll
        for (int k = 0; k < 8; ++k)
          pk[16 + k] = pack_bf16x2(ex2_mufu(fmaf(__uint_as_float(sb[2 * k]), c, -nu)),
                                   ex2_mufu(fmaf(__uint_as_float(sb[2 * k + 1]), c, -nu)));
#pragma unroll
        for (int k = 8; k < 16; ++k) pk[16 + k] = 0u;
      } else {
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          pk[k] = (2 * k < cn) ? pack_bf16x2(ex2_mufu(fmaf(__uint_as_float(sa[2 * k]), c, -nu)),
                                             ex2_mufu(fmaf(__uint_as_float(sa[2 * k + 1]), c, -nu)))
                               : 0u;
          pk[16 + k] = 0u;
        }
      }
      // P was last read by the value MMA of chunk q-1
      if (qq >= 1 && !mbar_wait_warp(p_free, (qq - 1) & 1, wc)) { ok = false; break; }
      tc_fence_after();
      tmem_st32(lane_base + Cfg::COL_P, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive_warp(p_full);
      if (cc == 0 && tile >= 1 && !epilogue(tile - 1)) { ok = false; break; }
    }
    if (ok && ntiles > 0) epilogue(ntiles - 1);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::TMEM_COLS);
  }
}

}  // namespace

size_t decode_smem_bytes(int D, int /*M*/) {
  const size_t need = (D == 16 ? DecCfg<16>::BYTES : DecCfg<32>::BYTES) + 1024;
  // at most dec_ctas_per_sm(D) CTAs per SM (TMEM columns)
  const size_t floor = dec_ctas_per_sm(D) >= 3 ? 70 * 1024 : 100 * 1024;
  return need > floor ? need : floor;
}

cudaError_t launch_decode(const CUtensorMap& tm_q, const CUtensorMap& tm_z, const CUtensorMap& tm_k,
                          const DecodeParams& p, cudaStream_t s) {
  const size_t smem = decode_smem_bytes(p.D, p.M);
  const dim3 grid(static_cast<unsigned>(p.B * p.H * p.ctas_per_head));
  if (p.D == 16) {
    cudaError_t e = cudaFuncSetAttribute(decode_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    decode_kernel<16><<<grid, DecCfg<16>::THREADS, smem, s>>>(tm_q, tm_z, tm_k, p);
  } else {
    cudaError_t e = cudaFuncSetAttribute(decode_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    decode_kernel<32><<<grid, DecCfg<32>::THREADS, smem, s>>>(tm_q, tm_z, tm_k, p);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (p.D == 16) decode_fallback_kernel<16><<<kNumSM, 128, 0, s>>>(p);
  else decode_fallback_kernel<32><<<kNumSM, 128, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace flare
