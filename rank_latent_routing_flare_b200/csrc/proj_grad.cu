// Projection gradients of the FLARE++ backward on tcgen05 (FLARE++ paper,
// section "Method": eq. 7 and eq. 9 run backwards).  With G the token-major
// gradient rows [R][4C] = [dK | dV | dK~ | dV~] (R = B*N tokens) and
// Wcat = [W_K | W_V | W~_K | W~_V] (each [C][C], K = X W_K):
//   dX = G Wcat^T               (dx_tc_kernel)
//   dWcat = X^T G               (dw_tc_kernel: per-split partials of its
//                                transpose, then dw_tc_reduce_kernel sums
//                                them in a fixed order)
// G arrives as two bf16 planes, high and low parts (G = Ghi + Glo to about
// 2^-16 relative), so every product runs as two kind::f16 MMAs on operands
// the tensor core reads straight from their bf16 storage (X and W are bf16
// already) with fp32 accumulation in TMEM.
//
// Both kernels stream 128-byte-wide (64 bf16) SW128 boxes through a TMA ring;
// one TMA box of G serves as a K-major operand (dX: rows are tokens, K = j)
// or as an MN-major one (dW^T: M = j, K = tokens).  Warp roles: warp 0 = TMA
// producer, warp 1 = MMA issuer + TMEM owner, warps 2..5 = epilogue (thread
// <-> TMEM lane).  Every wait is bounded (see ptx.cuh).
#include "bwd_internal.h"
#include "ptx.cuh"

namespace flare {
namespace {

constexpr int kPgBox = 64;  // bf16 elements in a 128-byte swizzle row

template <int C>
struct DxTcCfg {
  static constexpr int TR = 128;                   // token rows per tile
  static constexpr int A_B = TR * kPgBox * 2;      // one part of a G chunk (16 KB)
  static constexpr int W_B = C * kPgBox * 2;       // a [C][64] chunk of one W
  static constexpr int ST_B = 2 * A_B + W_B;       // Ghi, Glo, W
  static constexpr int NST = C == 256 ? 3 : 4;
  static constexpr int NCH = 4 * C / kPgBox;       // j chunks per tile
  static constexpr int OFF_BAR = NST * ST_B;
  static constexpr int OFF_MISC = OFF_BAR + 8 * 16;
  static constexpr int BYTES = OFF_MISC + 64;
  static constexpr uint32_t TMEM_COLS = 2 * C;     // two accumulators of C columns
  static_assert(ST_B % 1024 == 0, "ring stages start on a swizzle atom");
};

template <int C>
__global__ void __launch_bounds__(192, 1)
    dx_tc_kernel(const __grid_constant__ CUtensorMap tm_ghi, const __grid_constant__ CUtensorMap tm_glo,
                 const __grid_constant__ CUtensorMap tm_w0, const __grid_constant__ CUtensorMap tm_w1,
                 const __grid_constant__ CUtensorMap tm_w2, const __grid_constant__ CUtensorMap tm_w3,
                 const DxTcParams p) {
  using Cfg = DxTcCfg<C>;
  constexpr int NST = Cfg::NST, NCH = Cfg::NCH, KPW = C / kPgBox;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = sm;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Cfg::OFF_BAR);
  uint64_t* full = bars;                 // [NST] stage landed
  uint64_t* empty = bars + NST;          // [NST] stage read by its MMAs
  uint64_t* acc_full = bars + 2 * NST;   // [2] accumulator complete
  uint64_t* acc_free = acc_full + 2;     // [2] accumulator read by the epilogue
  uint64_t* mma_done = acc_free + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + Cfg::OFF_MISC);
  int* abort_flag = reinterpret_cast<int*>(sm + Cfg::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = (p.R + Cfg::TR - 1) / Cfg::TR;
  const int my_tiles = static_cast<int>(blockIdx.x) < n_tiles ? (n_tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  pdl_launch_dependents();
  if (my_tiles == 0) {
    pdl_wait();
    return;
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < NST; ++i) {
      mbar_init(full + i, 1);
      mbar_init(empty + i, 1);
    }
    for (int j = 0; j < 2; ++j) {
      mbar_init(acc_full + j, 1);
      mbar_init(acc_free + j, 4);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx wc{p.err, abort_flag, p.timeout_ns};

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tm_ghi);
      tma_prefetch_desc(&tm_glo);
      int issued = 0;
      for (int i = 0; i < my_tiles; ++i) {
        const int r0 = (blockIdx.x + i * gridDim.x) * Cfg::TR;
        bool ok = true;
        for (int jc = 0; jc < NCH; ++jc) {
          const int x = i * NCH + jc, st = x % NST;
          if (!mbar_wait(empty + st, ((x / NST) & 1) ^ 1, wc)) { ok = false; break; }
          uint8_t* dst = ring + st * Cfg::ST_B;
          mbar_arrive_expect_tx(full + st, Cfg::ST_B);
          tma_load_2d(dst, &tm_ghi, full + st, jc * kPgBox, r0);
          tma_load_2d(dst + Cfg::A_B, &tm_glo, full + st, jc * kPgBox, r0);
          // W_q rows c = 0..C-1, columns j0..j0+63 (each branch names its own
          // kernel parameter, so the map is read from parameter space)
          const int q = jc / KPW, j0 = (jc % KPW) * kPgBox;
          uint8_t* dw = dst + 2 * Cfg::A_B;
          switch (q) {
            case 0: tma_load_2d(dw, &tm_w0, full + st, j0, 0); break;
            case 1: tma_load_2d(dw, &tm_w1, full + st, j0, 0); break;
            case 2: tma_load_2d(dw, &tm_w2, full + st, j0, 0); break;
            default: tma_load_2d(dw, &tm_w3, full + st, j0, 0); break;
          }
          issued = x + 1;
        }
        if (!ok) break;
      }
      for (int x = max(0, issued - NST); x < issued; ++x)
        mbar_wait_drain(full + (x % NST), (x / NST) & 1, p.timeout_ns);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, C, false, false);
      const uint32_t ring_a = smem_u32(ring);
      bool ok = true;
      for (int i = 0; ok && i < my_tiles; ++i) {
        const int ab = i & 1;
        if (i >= 2 && !mbar_wait(acc_free + ab, ((i >> 1) - 1) & 1, wc)) break;
        tc_fence_after();
        for (int jc = 0; jc < NCH; ++jc) {
          const int x = i * NCH + jc, st = x % NST;
          if (!mbar_wait(full + st, (x / NST) & 1, wc)) { ok = false; break; }
          tc_fence_after();
          const uint32_t base = ring_a + st * Cfg::ST_B;
#pragma unroll
          for (int ks = 0; ks < kPgBox / 16; ++ks) {
            // K-major SW128: a k-step of 16 columns is 32 bytes inside the row
            const uint64_t ahi = umma_desc(base + ks * 32, 16, 1024, LAYOUT_SW128);
            const uint64_t alo = umma_desc(base + Cfg::A_B + ks * 32, 16, 1024, LAYOUT_SW128);
            const uint64_t bw = umma_desc(base + 2 * Cfg::A_B + ks * 32, 16, 1024, LAYOUT_SW128);
            umma_ss(tmem + ab * C, ahi, bw, idesc, (jc > 0 || ks > 0) ? 1u : 0u);
            umma_ss(tmem + ab * C, alo, bw, idesc, 1u);
          }
          umma_commit(empty + st);
        }
        if (!ok) break;
        umma_commit(acc_full + ab);
      }
      umma_commit(mma_done);
      mbar_wait_drain(mma_done, 0, p.timeout_ns);
    }
  } else {
    const int wq = warp & 3;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    for (int i = 0; i < my_tiles; ++i) {
      const int ab = i & 1;
      const long r = static_cast<long>(blockIdx.x + i * gridDim.x) * Cfg::TR + wq * 32 + lane;
      if (!mbar_wait_warp(acc_full + ab, (i >> 1) & 1, wc)) break;
      tc_fence_after();
#pragma unroll
      for (int c0 = 0; c0 < C; c0 += 64) {
        uint32_t v[64];
        tmem_ld32(lane_base + ab * C + c0, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
        tmem_ld32(lane_base + ab * C + c0 + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
        tmem_wait_ld();
        if (r < p.R) {
          uint4* dst = reinterpret_cast<uint4*>(p.dx + r * C + c0);
#pragma unroll
          for (int u = 0; u < 8; ++u)
            dst[u] = make_uint4(pack_bf16x2(__uint_as_float(v[8 * u]), __uint_as_float(v[8 * u + 1])),
                                pack_bf16x2(__uint_as_float(v[8 * u + 2]), __uint_as_float(v[8 * u + 3])),
                                pack_bf16x2(__uint_as_float(v[8 * u + 4]), __uint_as_float(v[8 * u + 5])),
                                pack_bf16x2(__uint_as_float(v[8 * u + 6]), __uint_as_float(v[8 * u + 7])));
        }
      }
      tc_fence_before();
      mbar_arrive_warp(acc_free + ab);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::TMEM_COLS);
  }
}

template <int C>
struct DwTcCfg {
  static constexpr int KR = 32;                    // token rows per chunk (two k-steps)
  static constexpr int JB = 256;                   // j per CTA: two M-tiles of 128
  static constexpr int BOX = KR * kPgBox * 2;      // one [32 rows][64] box (4 KB)
  static constexpr int G_B = (JB / kPgBox) * BOX;  // one part of the G chunk (16 KB)
  static constexpr int X_B = (C / kPgBox) * BOX;   // the X chunk
  static constexpr int ST_B = 2 * G_B + X_B;       // Ghi, Glo, X
  static constexpr int NST = 4;
  static constexpr int OFF_BAR = NST * ST_B;
  static constexpr int OFF_MISC = OFF_BAR + 8 * 16;
  static constexpr int BYTES = OFF_MISC + 64;
  static constexpr uint32_t TMEM_COLS = 2 * C;     // the two M-tiles' accumulators
  static_assert(BOX % 1024 == 0 && ST_B % 1024 == 0, "boxes start on a swizzle atom");
};

// part[s][j][c] = sum over the split's token rows r of G[r][j] X[r][c], for
// j in the CTA's block of 256: the transpose of X^T G, so that both operands
// are MN-major views of the token-major tiles (A = G^T: M = j, B = X^T: N = c,
// K = tokens).
template <int C>
__global__ void __launch_bounds__(192, 1)
    dw_tc_kernel(const __grid_constant__ CUtensorMap tm_ghi, const __grid_constant__ CUtensorMap tm_glo,
                 const __grid_constant__ CUtensorMap tm_x, const DwTcParams p) {
  using Cfg = DwTcCfg<C>;
  constexpr int NST = Cfg::NST, NJA = Cfg::JB / kPgBox, NXA = C / kPgBox;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = sm;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Cfg::OFF_BAR);
  uint64_t* full = bars;
  uint64_t* empty = bars + NST;
  uint64_t* acc_full = bars + 2 * NST;
  uint64_t* mma_done = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + Cfg::OFF_MISC);
  int* abort_flag = reinterpret_cast<int*>(sm + Cfg::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_jb = 4 * C / Cfg::JB;
  const int split = blockIdx.x / n_jb, jb = blockIdx.x % n_jb;
  const long rs = static_cast<long>(split) * p.rows_per_split;
  const long re = min(rs + p.rows_per_split, static_cast<long>(p.R));
  const int nch = re > rs ? static_cast<int>((re - rs + Cfg::KR - 1) / Cfg::KR) : 0;
  pdl_launch_dependents();
  if (threadIdx.x == 0) {
    for (int i = 0; i < NST; ++i) {
      mbar_init(full + i, 1);
      mbar_init(empty + i, 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx wc{p.err, abort_flag, p.timeout_ns};

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tm_ghi);
      tma_prefetch_desc(&tm_glo);
      tma_prefetch_desc(&tm_x);
      int issued = 0;
      for (int x = 0; x < nch; ++x) {
        const int st = x % NST;
        if (!mbar_wait(empty + st, ((x / NST) & 1) ^ 1, wc)) break;
        uint8_t* dst = ring + st * Cfg::ST_B;
        const int r0 = static_cast<int>(rs) + x * Cfg::KR;
        mbar_arrive_expect_tx(full + st, Cfg::ST_B);
        for (int a = 0; a < NJA; ++a) {
          const int j0 = jb * Cfg::JB + a * kPgBox;
          tma_load_2d(dst + a * Cfg::BOX, &tm_ghi, full + st, j0, r0);
          tma_load_2d(dst + Cfg::G_B + a * Cfg::BOX, &tm_glo, full + st, j0, r0);
        }
        for (int a = 0; a < NXA; ++a) tma_load_2d(dst + 2 * Cfg::G_B + a * Cfg::BOX, &tm_x, full + st, a * kPgBox, r0);
        issued = x + 1;
      }
      for (int x = max(0, issued - NST); x < issued; ++x)
        mbar_wait_drain(full + (x % NST), (x / NST) & 1, p.timeout_ns);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, C, true, true);
      const uint32_t ring_a = smem_u32(ring);
      bool ok = true;
      for (int x = 0; x < nch; ++x) {
        const int st = x % NST;
        if (!mbar_wait(full + st, (x / NST) & 1, wc)) { ok = false; break; }
        tc_fence_after();
        const uint32_t base = ring_a + st * Cfg::ST_B;
#pragma unroll
        for (int ks = 0; ks < Cfg::KR / 16; ++ks) {
          // MN-major SW128: a k-step of 16 rows is 16 x 128 bytes; the 64-wide
          // atoms of M (or N) are one box apart, 8-row groups 1024 bytes apart
          const uint64_t bx = umma_desc(base + 2 * Cfg::G_B + ks * 16 * 128, Cfg::BOX, 1024, LAYOUT_SW128);
#pragma unroll
          for (int m = 0; m < 2; ++m) {
            const uint32_t goff = m * 2 * Cfg::BOX + ks * 16 * 128;
            const uint64_t ahi = umma_desc(base + goff, Cfg::BOX, 1024, LAYOUT_SW128);
            const uint64_t alo = umma_desc(base + Cfg::G_B + goff, Cfg::BOX, 1024, LAYOUT_SW128);
            umma_ss(tmem + m * C, ahi, bx, idesc, (x > 0 || ks > 0) ? 1u : 0u);
            umma_ss(tmem + m * C, alo, bx, idesc, 1u);
          }
        }
        umma_commit(empty + st);
      }
      if (ok && nch > 0) umma_commit(acc_full);
      umma_commit(mma_done);
      mbar_wait_drain(mma_done, 0, p.timeout_ns);
    }
  } else {
    const int wq = warp & 3;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const bool have = nch > 0 && mbar_wait_warp(acc_full, 0, wc);
    if (have) tc_fence_after();
    if (nch == 0 || have) {
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        const int j = jb * Cfg::JB + m * 128 + wq * 32 + lane;
        float* row = p.part + (static_cast<size_t>(split) * 4 * C + j) * C;
#pragma unroll
        for (int c0 = 0; c0 < C; c0 += 32) {
          uint32_t v[32];
          if (have) {
            tmem_ld32(lane_base + m * C + c0, v);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int u = 0; u < 32; ++u) v[u] = 0u;
          }
          float4* dst = reinterpret_cast<float4*>(row + c0);
#pragma unroll
          for (int u = 0; u < 8; ++u)
            dst[u] = make_float4(__uint_as_float(v[4 * u]), __uint_as_float(v[4 * u + 1]),
                                 __uint_as_float(v[4 * u + 2]), __uint_as_float(v[4 * u + 3]));
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

// dW_q[c][jj] = sum over the splits of part[s][q*C + jj][c] (+ the (q+2)
// block when the synthesis weights are the encode weights).  A block of 256
// threads owns 32 consecutive c of one row j: its eight warps sum the splits
// w, w + 8, w + 16, ... (lanes along c, so the reads coalesce) and the eight
// partial sums are then added in warp order: a fixed order, so the result
// does not depend on timing.
constexpr int kRedGroups = 8;

__global__ void __launch_bounds__(256) dw_tc_reduce_kernel(const DwReduceParams p) {
  __shared__ float red[kRedGroups][32];
  const int cblocks = p.C / 32;
  const int j = blockIdx.x / cblocks;
  const int lane = threadIdx.x & 31, g = threadIdx.x >> 5;
  const int c = (blockIdx.x % cblocks) * 32 + lane;
  float s = 0.f;
  for (int sp = g; sp < p.n_splits; sp += kRedGroups) {
    const float* blk = p.part + static_cast<size_t>(sp) * p.J * p.C;
    s += blk[static_cast<size_t>(j) * p.C + c];
    if (p.shared) s += blk[static_cast<size_t>(j + 2 * p.C) * p.C + c];
  }
  red[g][lane] = s;
  __syncthreads();
  if (g != 0) return;
  float t = red[0][lane];
#pragma unroll
  for (int k = 1; k < kRedGroups; ++k) t += red[k][lane];
  const int q = j / p.C, jj = j % p.C;
  if (p.dw[q]) p.dw[q][static_cast<size_t>(c) * p.C + jj] = t;
  if (p.shared && p.dw[q + 2]) p.dw[q + 2][static_cast<size_t>(c) * p.C + jj] = t;
}

template <class Cfg>
size_t pg_smem() {
  return Cfg::BYTES + 1024;
}

}  // namespace

cudaError_t launch_dx_tc(const DxTcMaps& m, const DxTcParams& p, cudaStream_t s) {
  const int n_tiles = (p.R + 127) / 128;
  const unsigned grid = static_cast<unsigned>(std::min(n_tiles, kNumSM));
  auto go = [&](auto kern, size_t smem) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    kern<<<grid, 192, smem, s>>>(m.ghi, m.glo, m.w[0], m.w[1], m.w[2], m.w[3], p);
    return cudaGetLastError();
  };
  switch (p.C) {
    case 64: return go(dx_tc_kernel<64>, pg_smem<DxTcCfg<64>>());
    case 128: return go(dx_tc_kernel<128>, pg_smem<DxTcCfg<128>>());
    case 256: return go(dx_tc_kernel<256>, pg_smem<DxTcCfg<256>>());
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_dw_tc(const DwTcMaps& m, const DwTcParams& p, cudaStream_t s) {
  const unsigned grid = static_cast<unsigned>(p.n_splits * (4 * p.C / 256));
  auto go = [&](auto kern, size_t smem) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    kern<<<grid, 192, smem, s>>>(m.ghi, m.glo, m.x, p);
    return cudaGetLastError();
  };
  switch (p.C) {
    case 64: return go(dw_tc_kernel<64>, pg_smem<DwTcCfg<64>>());
    case 128: return go(dw_tc_kernel<128>, pg_smem<DwTcCfg<128>>());
    case 256: return go(dw_tc_kernel<256>, pg_smem<DwTcCfg<256>>());
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_dw_tc_reduce(const DwReduceParams& p, cudaStream_t s) {
  if (p.C % 32 != 0) return cudaErrorInvalidValue;
  const long rows = p.shared ? 2 * p.C : p.J;
  dw_tc_reduce_kernel<<<static_cast<unsigned>(rows * (p.C / 32)), kRedGroups * 32, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace flare
