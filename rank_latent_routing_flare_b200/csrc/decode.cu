// Decoder SDPA on tcgen05 (FLARE++ paper, arXiv 2608.11519, section "Method":
// the FLARE decoder Y_h = softmax_m(K_h Q_h^T / sqrt(D)) Z_h of eq. 6, used
// with Q_h(X) in eq. 11).
//
// One CTA owns one head (b, h) and a contiguous range of 128-token tiles.  The
// head's queries Q (M x D) and latent values Z (M x D) stay resident in shared
// memory; key tiles stream through a TMA ring.  Per tile and per chunk of C
// latents (C = dec_chunk(D); the last chunk may be shorter):
//   S = K_tile Q_c^T               UMMA M=128 (tokens) x N=C (latents), fp32 TMEM
//   P = 2^(S * c - nu_n)           softmax threads, one token row per thread
//   Y += P [Z_c | 1]               UMMA with A = P read from TMEM; column D of Y
//                                  accumulates the row sum
// nu_n = c * |k_n| * max_m |q_m| bounds the token's scaled scores from above
// (Cauchy-Schwarz), so the latent chunks need no running maximum.  A token
// whose sum underflows (only possible when the bound is very loose) is listed
// and recomputed exactly by decode_fallback_kernel.
//
// The chunks of all tiles form one sequence q = tile * nc + chunk.  TMEM holds
// NB score buffers (dec_bufs: two at D = 16, three at D = 32; chunk q uses
// buffer q % NB; the softmax threads write P_q over the first C/2 columns of
// S_q once S_q is in registers) and the Y accumulator.  The MMA thread issues
// S_{q+2} right after P_q [Z_c | 1] (with two buffers, once that value MMA is
// done; with three, at once, since S_{q+2}'s buffer last held P_{q-1}), so
// the softmax threads find S_{q+1} ready when they finish chunk q.  Every
// barrier reused across chunks exists once per buffer, so no party can run a
// full phase ahead of the party that waits on it.  The epilogue of a tile
// (Y / sum, bf16 stores) runs after the first chunk of the next tile.
//
// With F16 (the training forward, D = 16) the value product runs on fp16
// operands: Z as fp16 (11-bit mantissa instead of bf16's 8) and the weights
// as fp16 P' = 2^(S c - nu + 14), scaled by 2^14 so that weights down to
// 2^-28 of the bound keep full fp16 precision (the scale cancels in Y = acc /
// sum).  Y, and the fp32 copy the backward takes delta_n from, then see Z to
// 2^-12; the epilogue also writes L_n.  Rows whose scaled sum falls below
// 2^-14 (a bound looser than 28 in log2 units) go to the exact fallback.
//
// Warp roles (5 warps): warp 0 lane 0 is the MMA thread (it also loads Q, Z
// and the first key tiles).  Warps 1..4 are the softmax warps (thread <->
// TMEM lane <-> token); one of them, in rotation, refills the key ring.  A
// CTA needs 128 TMEM columns for D = 16 (two 48-latent score buffers and Y),
// so four CTAs share an SM.
#include <type_traits>

#include "ptx.cuh"

namespace flare {
namespace {

template <int D, bool F16>
struct DecCfg {
  static_assert(!F16 || D == 16, "the fp16 value product is built for D = 16 only");
  static constexpr int C = dec_chunk(D);                // latents per chunk
  static constexpr int ROWB = D * 2;
  static constexpr int KT_B = kDecTile * ROWB;          // one key tile
  static constexpr int QZ_B = 512 * ROWB;               // all of Q (or Z): M <= 512
  static constexpr int NST = 4;                         // key ring stages
  static constexpr uint32_t LAYOUT = (D == 16) ? LAYOUT_SW32 : LAYOUT_SW64;
  static constexpr uint32_t SBO = 8 * ROWB;
  static constexpr int NY = D + 16;                     // Y columns: D values + sums
  static constexpr int NB = dec_bufs(D);                // score buffers
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_Z = OFF_Q + QZ_B;
  static constexpr int OFF_ONES = OFF_Z + QZ_B;         // C x ROWB block of ones
  static constexpr int OFF_K = OFF_ONES + C * ROWB;     // NST * KT_B
  static constexpr int OFF_BAR = OFF_K + NST * KT_B;
  static constexpr int OFF_MISC = OFF_BAR + 8 * (4 + NST + 3 * NB);
  static constexpr int BYTES = OFF_MISC + 64 + NST * 4;
  // TMEM columns: score buffers at 0, C, 2C (each later holds its P), Y at 3C
  static constexpr uint32_t COL_Y = NB * C;
  static constexpr uint32_t TMEM_COLS = (COL_Y + NY <= 128) ? 128 : 256;
  static constexpr int THREADS = 160;
  static constexpr int CTAS_PER_SM = dec_ctas_per_sm(D);
  static_assert(TMEM_COLS <= 512 / CTAS_PER_SM, "TMEM columns of the co-resident CTAs exceed 512");
  static_assert(COL_Y + NY <= TMEM_COLS, "score buffers and Y exceed the allocation");
  static_assert(OFF_K % 512 == 0 || D == 16, "key tiles must start on a swizzle atom");
  static_assert(OFF_K % 256 == 0, "key tiles must start on a swizzle atom");
};

// Output row of token n of head bh: [B*H][N][D], or [B][N][H*D] (the heads of
// a token side by side) when p.y_token_major.
template <int D>
__device__ __forceinline__ uint16_t* y_row(const DecodeParams& p, int bh, int n) {
  if (p.y_token_major) {
    const int b = bh / p.H, h = bh - b * p.H;
    return p.y + (static_cast<size_t>(b) * p.N + n) * (static_cast<size_t>(p.H) * D) + static_cast<size_t>(h) * D;
  }
  return p.y + (static_cast<size_t>(bh) * p.N + n) * D;
}

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
  pdl_wait();
  const uint32_t count = *p.fb_count;
  for (uint32_t e = blockIdx.x * blockDim.x + threadIdx.x; e < count; e += gridDim.x * blockDim.x) {
    const uint64_t tok = p.fb_list[e];
    const int bh = static_cast<int>(tok / static_cast<uint64_t>(p.N));
    const int n = static_cast<int>(tok % static_cast<uint64_t>(p.N));
    const int g = p.q_per_batch ? bh : bh % p.H;
    const uint16_t* krow = p.k + (static_cast<size_t>(bh) * p.N + n) * D;
    const uint16_t* qg = p.q + static_cast<size_t>(g) * p.M * D;
    const uint16_t* zh = p.z + static_cast<size_t>(bh) * p.M * D;
    const float* zf = p.z32 != nullptr ? p.z32 + static_cast<size_t>(bh) * p.M * D : nullptr;
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
      if (zf != nullptr) {
#pragma unroll
        for (int d = 0; d < D; ++d) y[d] = fmaf(w, zf[m * D + d], y[d]);
      } else {
#pragma unroll
        for (int d = 0; d < D; ++d) y[d] = fmaf(w, __uint_as_float(static_cast<uint32_t>(zh[m * D + d]) << 16), y[d]);
      }
    }
    const float inv = 1.f / den;
    if (p.ltok_out != nullptr) p.ltok_out[static_cast<size_t>(bh) * p.N + n] = mx + log2f(den);
    if (p.y_f32 != nullptr) {
      float4* d32 = reinterpret_cast<float4*>(p.y_f32 + (static_cast<size_t>(bh) * p.N + n) * D);
#pragma unroll
      for (int u = 0; u < D / 4; ++u)
        d32[u] = make_float4(y[4 * u] * inv, y[4 * u + 1] * inv, y[4 * u + 2] * inv, y[4 * u + 3] * inv);
    }
    if (p.y == nullptr) continue;
    uint4* dst = reinterpret_cast<uint4*>(y_row<D>(p, bh, n));
#pragma unroll
    for (int u = 0; u < D / 8; ++u)
      dst[u] = make_uint4(pack_bf16x2(y[8 * u + 0] * inv, y[8 * u + 1] * inv),
                          pack_bf16x2(y[8 * u + 2] * inv, y[8 * u + 3] * inv),
                          pack_bf16x2(y[8 * u + 4] * inv, y[8 * u + 5] * inv),
                          pack_bf16x2(y[8 * u + 6] * inv, y[8 * u + 7] * inv));
  }
}

template <int D, bool F16>
__global__ void __launch_bounds__(DecCfg<D, F16>::THREADS, DecCfg<D, F16>::CTAS_PER_SM)
    decode_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_z,
                  const __grid_constant__ CUtensorMap tm_k, const DecodeParams p) {
  using Cfg = DecCfg<D, F16>;
  constexpr int NST = Cfg::NST, C = Cfg::C, NB = Cfg::NB;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sq = sm + Cfg::OFF_Q;
  uint8_t* sz = sm + Cfg::OFF_Z;
  uint8_t* sones = sm + Cfg::OFF_ONES;
  uint8_t* sk = sm + Cfg::OFF_K;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Cfg::OFF_BAR);
  uint64_t* qz_full = bars;
  uint64_t* k_full = bars + 1;             // [NST] key tile landed
  uint64_t* s_full = bars + 1 + NST;       // [NB] score buffer computed
  uint64_t* pv_done = s_full + NB;         // [NB] value MMA done reading the buffer's P
  uint64_t* p_full = s_full + 2 * NB;      // [NB] P stored by every softmax warp
  uint64_t* y_full = s_full + 3 * NB;      // Y of a tile complete
  uint64_t* y_free = y_full + 1;           // Y read by every softmax warp
  uint64_t* mma_done = y_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + Cfg::OFF_MISC);
  int* abort_flag = reinterpret_cast<int*>(sm + Cfg::OFF_MISC + 4);
  float* red = reinterpret_cast<float*>(sm + Cfg::OFF_MISC + 16);
  volatile int* last_load = reinterpret_cast<volatile int*>(sm + Cfg::OFF_MISC + 64);  // per stage

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.x / p.ctas_per_head;
  const int part = blockIdx.x % p.ctas_per_head;
  const int b = bh / p.H, h = bh % p.H;
  const int g = p.q_per_batch ? bh : h;
  bool bad_len = false;
  const int L = shard_valid_len(p.lengths, b, p.N, p.tok_offset, p.n_global, &bad_len);
  if (bad_len && threadIdx.x == 0) atomicOr(p.err, FLARE_DEV_BAD_LENGTH);
  const int tiles_head = (p.N + kDecTile - 1) / kDecTile;
  const int tiles_valid = (L + kDecTile - 1) / kDecTile;
  const int ta = part * p.tiles_per_cta;
  const int tb = min(ta + p.tiles_per_cta, tiles_head);
  const int tc_end = min(tb, tiles_valid);            // tiles [ta, tc_end) are computed
  const int ntiles = max(0, tc_end - ta);
  const int nc = (p.M + C - 1) / C;                   // latent chunks
  pdl_launch_dependents();

  // tiles entirely past the valid length: zero rows
  auto zero_rows = [&]() {
    const int z0 = max(ta, tiles_valid) * kDecTile;
    const int z1 = min(tb * kDecTile, p.N);
    const uint4 zero = make_uint4(0, 0, 0, 0);
    if (p.y != nullptr)
      for (size_t e = static_cast<size_t>(z0) * (D / 8) + threadIdx.x; e < static_cast<size_t>(z1) * (D / 8);
           e += blockDim.x)
        reinterpret_cast<uint4*>(y_row<D>(p, bh, static_cast<int>(e / (D / 8))))[e % (D / 8)] = zero;
    if (p.y_f32 != nullptr) {
      uint4* d32 = reinterpret_cast<uint4*>(p.y_f32 + static_cast<size_t>(bh) * p.N * D);
      for (size_t e = static_cast<size_t>(z0) * (D / 4) + threadIdx.x; e < static_cast<size_t>(z1) * (D / 4);
           e += blockDim.x)
        d32[e] = zero;
    }
  };
  if (ntiles == 0) {
    pdl_wait();
    zero_rows();
    return;
  }

  if (threadIdx.x == 0) {
    mbar_init(qz_full, 1);
    for (int i = 0; i < NST; ++i) {
      mbar_init(k_full + i, 1);
      last_load[i] = -1;
    }
    for (int i = 0; i < NB; ++i) {
      mbar_init(s_full + i, 1);
      mbar_init(pv_done + i, 1);
      mbar_init(p_full + i, 4);
    }
    mbar_init(y_full, 1);
    mbar_init(y_free, 4);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  for (int i = threadIdx.x; i < C * Cfg::ROWB / 4; i += blockDim.x)
    reinterpret_cast<uint32_t*>(sones)[i] = F16 ? 0x3C003C00u : 0x3F803F80u;  // 1.0 pairs (fp16 or bf16)
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
  zero_rows();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx wc{p.err, abort_flag, p.timeout_ns};
  // key tile n (of this CTA's range) into ring stage n % NST (one thread)
  auto load_tile = [&](int n) {
    const int st = n % NST;
    mbar_arrive_expect_tx(k_full + st, Cfg::KT_B);
    tma_load_3d(sk + st * Cfg::KT_B, &tm_k, k_full + st, 0, (ta + n) * kDecTile, bh);
    last_load[st] = n;
  };
  const int total = ntiles * nc;

  if (warp == 0) {
    // ------------------------------------------------------------ MMA thread
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_z);
      tma_prefetch_desc(&tm_k);
      const int nbox = (p.M + p.qz_box_rows - 1) / p.qz_box_rows;
      mbar_arrive_expect_tx(qz_full, 2 * nbox * p.qz_box_rows * Cfg::ROWB);
      for (int bx = 0; bx < nbox; ++bx) {
        tma_load_3d(sq + bx * p.qz_box_rows * Cfg::ROWB, &tm_q, qz_full, 0, bx * p.qz_box_rows, g);
        tma_load_3d(sz + bx * p.qz_box_rows * Cfg::ROWB, &tm_z, qz_full, 0, bx * p.qz_box_rows, bh);
      }
      for (int n = 0; n < min(NST, ntiles); ++n) load_tile(n);
      const uint32_t idesc_y = F16 ? idesc_f16_f32(128, Cfg::NY, false, true) : idesc_bf16_f32(128, Cfg::NY, false, true);
      const uint32_t sz_a = smem_u32(sz), ones_a = smem_u32(sones);
      const uint64_t q_desc = umma_desc(smem_u32(sq), 16, Cfg::SBO, Cfg::LAYOUT);
      const uint64_t k_desc = umma_desc(smem_u32(sk), 16, Cfg::SBO, Cfg::LAYOUT);
      // chunk q = tile * nc + cc, tracked incrementally (no division per chunk)
      struct Cursor {
        int q, tile, cc;
      };
      auto advance = [&](Cursor& x) {
        ++x.q;
        if (++x.cc == nc) {
          x.cc = 0;
          ++x.tile;
        }
      };
      const int last_n = p.M - (nc - 1) * C;            // latents of the last chunk
      const uint32_t idesc_full = idesc_bf16_f32(128, C, false, false);
      const uint32_t idesc_last = idesc_bf16_f32(128, last_n, false, false);
      constexpr uint64_t CH_STEP = (C * Cfg::ROWB) >> 4;  // descriptor units per chunk
      // [Z_c | 1]: chunk c starts CH_STEP * c further on, and its ones block
      // (leading byte offset) is that much closer
      const uint64_t z_desc = umma_desc(sz_a, ones_a - sz_a, Cfg::SBO, Cfg::LAYOUT);
      // S_q = K_tile Q_c^T into buffer q % NB, once the key tile has landed and
      // P_{q-NB} has been consumed
      auto issue_s = [&](const Cursor& x) -> bool {
        const int buf = x.q % NB, st = x.tile % NST;
        if (x.cc == 0 && !mbar_wait_mma(k_full + st, (x.tile / NST) & 1, wc)) return false;
        if (x.q >= NB && !mbar_wait_mma(pv_done + buf, ((x.q - NB) / NB) & 1, wc)) return false;
        tc_fence_after();
        const uint32_t idesc_s = x.cc == nc - 1 ? idesc_last : idesc_full;
        const uint64_t kd = k_desc + static_cast<uint64_t>(st) * (Cfg::KT_B >> 4);
        const uint64_t qd = q_desc + static_cast<uint64_t>(x.cc) * CH_STEP;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          umma_ss(tmem + buf * C, kd + 2 * kk, qd + 2 * kk, idesc_s, kk > 0 ? 1u : 0u);
        umma_commit(s_full + buf);
        return true;
      };
      // Y += P_q [Z_c | 1] once every softmax warp has stored P_q (and, for a
      // tile's first chunk, has read the previous tile's Y)
      auto issue_pv = [&](const Cursor& x) -> bool {
        const int buf = x.q % NB;
        if (!mbar_wait_mma(p_full + buf, (x.q / NB) & 1, wc)) return false;
        if (x.cc == 0 && x.tile >= 1 && !mbar_wait_mma(y_free, (x.tile - 1) & 1, wc)) return false;
        tc_fence_after();
        const uint64_t step = static_cast<uint64_t>(x.cc) * CH_STEP;
        const uint64_t zd = z_desc + step - (step << 16);
        const int nks = (x.cc == nc - 1 ? last_n : C) / 16;
#pragma unroll
        for (int ks = 0; ks < C / 16; ++ks)
          if (ks < nks)
            umma_ts(tmem + Cfg::COL_Y, tmem + buf * C + ks * 8,
                    zd + static_cast<uint64_t>((ks * 16 * Cfg::ROWB) >> 4), idesc_y, (x.cc > 0 || ks > 0) ? 1u : 0u);
        umma_commit(pv_done + buf);
        if (x.cc == nc - 1) umma_commit(y_full);
        return true;
      };
      Cursor cs{0, 0, 0}, cp{0, 0, 0};
      bool ok = mbar_wait_mma(qz_full, 0, wc) && issue_s(cs);
      advance(cs);
      if (ok && total > 1) ok = issue_s(cs);
      advance(cs);
      for (; ok && cp.q < total; advance(cp)) {
        ok = issue_pv(cp);
        if (ok && cs.q < total) {
          ok = issue_s(cs);
          advance(cs);
        }
      }
      umma_commit(mma_done);  // every MMA issued above is complete before TMEM is freed
      mbar_wait_drain(mma_done, 0, p.timeout_ns);
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
    // (Reading Y before the next tile's first exponentials instead, so that
    // the next value MMA need not wait for it, measured 4 % slower.)
    auto epilogue = [&](int i, float nu_i) -> bool {
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
      // F16: the weights carry 2^14, and a sum below 2^-14 means weights in
      // fp16's subnormal range
      const bool exact = n < L && !(l >= (F16 ? 0x1p-14f : 0x1p-90f));
      if (n < L) {
        const float inv = 1.f / l;
#pragma unroll
        for (int d = 0; d < D; ++d) y[d] *= inv;
      } else {
#pragma unroll
        for (int d = 0; d < D; ++d) y[d] = 0.f;
      }
      if constexpr (F16) {  // L_n for the training backward (the weights carry 2^14)
        if (p.ltok_out != nullptr && n < p.N && !exact)
          p.ltok_out[static_cast<size_t>(bh) * p.N + n] = n < L ? nu_i - 14.f + log2f(l) : 0.f;
      }
      if (exact) {  // recomputed exactly by decode_fallback_kernel
        const uint32_t e = atomicAdd(p.fb_count, 1u);
        p.fb_list[e] = static_cast<uint64_t>(bh) * p.N + n;
      } else if (n < p.N) {
        if (p.y_f32 != nullptr) {
          float4* d32 = reinterpret_cast<float4*>(p.y_f32 + (static_cast<size_t>(bh) * p.N + n) * D);
#pragma unroll
          for (int u = 0; u < D / 4; ++u) d32[u] = make_float4(y[4 * u], y[4 * u + 1], y[4 * u + 2], y[4 * u + 3]);
        }
        if (p.y != nullptr) {
          uint4* dst = reinterpret_cast<uint4*>(y_row<D>(p, bh, n));
#pragma unroll
          for (int u = 0; u < D / 8; ++u)
            dst[u] = make_uint4(pack_bf16x2(y[8 * u + 0], y[8 * u + 1]), pack_bf16x2(y[8 * u + 2], y[8 * u + 3]),
                                pack_bf16x2(y[8 * u + 4], y[8 * u + 5]), pack_bf16x2(y[8 * u + 6], y[8 * u + 7]));
        }
      }
      return true;
    };
    // exponentials of one chunk of CN latents in buffer column base cb: the
    // first 16 columns are exponentiated while the rest are read from TMEM
    auto run_chunk = [&](auto cn_tag, uint32_t cb, float nu) {
      constexpr int CN = decltype(cn_tag)::value;
      const float nu_p = F16 ? nu - 14.f : nu;  // F16: weights scaled by 2^14
      uint32_t s0[16], pk[CN / 2];
      tmem_ld16(cb, s0);
      tmem_wait_ld();
      if constexpr (CN > 16) {
        uint32_t s1[CN - 16];
        tmem_ld_cols<CN - 16>(cb + 16, s1);
        exp2_row<16, FLARE_DEC_POLY_PAIRS, 0, F16>(s0, c, nu_p, *reinterpret_cast<uint32_t(*)[8]>(&pk[0]));
        tmem_wait_ld();
        exp2_row<CN - 16, FLARE_DEC_POLY_PAIRS, 8, F16>(s1, c, nu_p,
                                                   *reinterpret_cast<uint32_t(*)[(CN - 16) / 2]>(&pk[8]));
      } else {
        exp2_row<16, FLARE_DEC_POLY_PAIRS, 0, F16>(s0, c, nu_p, pk);
      }
      tmem_st_cols<CN / 2>(cb, pk);  // P over the first CN/2 columns of the chunk's scores
      tmem_wait_st();
    };
    bool ok = true;
    float nu = 0.f, nu_prev = 0.f;  // shift bounds of the current and the previous tile
    for (int q = 0, tile = 0, cc = 0, buf = 0, use = 0; q < total; ++q) {
      if (!mbar_wait_warp(s_full + buf, use & 1, wc)) { ok = false; break; }
      tc_fence_after();
      if (cc == 0) {
        // |k_n| from the key tile in shared memory (the swizzle only permutes
        // 16-byte pieces inside each row, which a sum of squares ignores); the
        // tile's stage is refilled only after every warp is past this point
        if (!mbar_wait_warp(k_full + tile % NST, (tile / NST) & 1, wc)) { ok = false; break; }
        const uint4* krow_s = reinterpret_cast<const uint4*>(sk + (tile % NST) * Cfg::KT_B + r * Cfg::ROWB);
        if constexpr (F16) nu_prev = nu;
        nu = c * sqrtf(bf16_row_norm2(krow_s, D / 8)) * qm;
      }
      const int cn = min(C, p.M - cc * C);
      const uint32_t cb = lane_base + buf * C;
      if (cn == C) run_chunk(std::integral_constant<int, C>{}, cb, nu);
      else if (C > 48 && cn == 48) run_chunk(std::integral_constant<int, (C > 48 ? 48 : 16)>{}, cb, nu);
      else if (C > 32 && cn == 32) run_chunk(std::integral_constant<int, (C > 32 ? 32 : 16)>{}, cb, nu);
      else run_chunk(std::integral_constant<int, 16>{}, cb, nu);
      tc_fence_before();
      mbar_arrive_warp(p_full + buf);
      if (cc == 0 && tile >= 2 && tile - 2 + NST < ntiles && wq == (tile & 3) && lane == 0)
        load_tile(tile - 2 + NST);  // every MMA and norm read of tile - 2 is done
      __syncwarp();
      if (cc == 0 && tile >= 1 && !epilogue(tile - 1, nu_prev)) { ok = false; break; }
      if (++cc == nc) {
        cc = 0;
        ++tile;
      }
      if (++buf == NB) {
        buf = 0;
        ++use;
      }
    }
    if (ok) epilogue(ntiles - 1, nu);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    if (lane == 0) {  // copies still in flight (only after an abort) must land before exit
      for (int st = 0; st < NST; ++st)
        if (last_load[st] >= 0) mbar_wait_drain(k_full + st, (last_load[st] / NST) & 1, p.timeout_ns);
      mbar_wait_drain(qz_full, 0, p.timeout_ns);
    }
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::TMEM_COLS);
  }
}

}  // namespace

size_t decode_smem_bytes(int D) {
  const size_t need = (D == 16 ? DecCfg<16, false>::BYTES : DecCfg<32, false>::BYTES) + 1024;
  // at most dec_ctas_per_sm(D) CTAs per SM (228 KB each, 1 KB of it
  // reserved per CTA), so that every resident CTA finds its TMEM columns free
  const size_t floor = (228 * 1024) / (dec_ctas_per_sm(D) + 1) + 1024;
  return need > floor ? need : floor;
}

cudaError_t launch_decode(const CUtensorMap& tm_q, const CUtensorMap& tm_z, const CUtensorMap& tm_k,
                          const DecodeParams& p, cudaStream_t s, bool pdl) {
  if (p.z_f16 && p.D != 16) return cudaErrorInvalidValue;
  const size_t smem = decode_smem_bytes(p.D);
  const dim3 grid(static_cast<unsigned>(p.B * p.H * p.ctas_per_head));
  auto go = [&](auto kern, int threads) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    LaunchCfg lc(grid, dim3(threads), smem, s, pdl);
    return cudaLaunchKernelEx(&lc.cfg, kern, tm_q, tm_z, tm_k, p);
  };
  cudaError_t e = p.D != 16 ? go(decode_kernel<32, false>, DecCfg<32, false>::THREADS)
                  : p.z_f16 ? go(decode_kernel<16, true>, DecCfg<16, true>::THREADS)
                            : go(decode_kernel<16, false>, DecCfg<16, false>::THREADS);
  if (e != cudaSuccess) return e;
  // the fallback follows the decoder on the same stream: always programmatic
  LaunchCfg fb(dim3(kNumSM), dim3(128), 0, s, true);
  return p.D == 16 ? cudaLaunchKernelEx(&fb.cfg, decode_fallback_kernel<16>, p)
                   : cudaLaunchKernelEx(&fb.cfg, decode_fallback_kernel<32>, p);
}

}  // namespace flare
