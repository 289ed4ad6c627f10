// Per-head projections K~ = X W~_K, V~ = X W~_V, K = X W_K, V = X W_V on
// tcgen05 (FLARE++ paper, arXiv 2608.11519, section "Method": eq. 7 and
// eq. 9; head h takes column block [h*D, (h+1)*D) of each C x C matrix as in
// section "Full self-attention").
//
// A CTA owns one projection p and a strided set of 128-token tiles.  W_p stays
// resident in shared memory (MN-major SW128 UMMA operand); X tiles stream in
// 64-column chunks (K-major SW128).  The fp32 accumulator (128 x C) lives in
// TMEM, double-buffered so that the epilogue of one tile overlaps the MMAs of
// the next.  The epilogue rounds to bf16, scatters to the [B][H][N][D] head
// layout and, for the two key projections, records the largest key norm of
// every 32-token group (used by the encoder as its softmax shift bound).
//
// Warp roles: warp 0 = TMA producer, warp 1 = MMA issuer + TMEM owner,
// warps 2..5 = epilogue (thread <-> TMEM lane <-> token).
#include "ptx.cuh"

namespace flare {
namespace {

// Largest value of a non-negative float across the warp: for v >= 0 the
// bit patterns order like the values, so one integer max reduction does it.
__device__ __forceinline__ float warp_max_nonneg(float v) {
  return __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(v)));
}

template <int C>
struct ProjCfg {
  static constexpr int KC = C / 64;                   // 64-wide K chunks
  static constexpr int W_BOX = 64 * 64 * 2;           // one 64x64 bf16 box
  static constexpr int W_B = KC * KC * W_BOX;         // whole W_p
  static constexpr int X_B = kProjTile * 64 * 2;      // one X chunk (128 tokens x 64)
  static constexpr int NST = 4;
  static constexpr int OFF_W = 0;
  static constexpr int OFF_X = OFF_W + W_B;
  static constexpr int OFF_BAR = OFF_X + NST * X_B;
  static constexpr int OFF_MISC = OFF_BAR + 8 * 32;
  static constexpr int BYTES = OFF_MISC + 64;
  static constexpr uint32_t TMEM_COLS = (2 * C < 32) ? 32 : 2 * C;  // two accumulators of C columns
};

template <int C, int D>
__global__ void __launch_bounds__(192, 1)
    project_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w0,
                   const __grid_constant__ CUtensorMap tm_w1, const __grid_constant__ CUtensorMap tm_w2,
                   const __grid_constant__ CUtensorMap tm_w3, const ProjParams p) {
  using Cfg = ProjCfg<C>;
  constexpr int NST = Cfg::NST, KC = Cfg::KC;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sw = sm + Cfg::OFF_W;
  uint8_t* sx = sm + Cfg::OFF_X;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Cfg::OFF_BAR);
  uint64_t* w_full = bars;
  uint64_t* x_full = bars + 1;
  uint64_t* x_empty = bars + 1 + NST;
  uint64_t* acc_full = bars + 1 + 2 * NST;
  uint64_t* acc_free = acc_full + 2;
  uint64_t* mma_done = acc_free + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + Cfg::OFF_MISC);
  int* abort_flag = reinterpret_cast<int*>(sm + Cfg::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int proj = blockIdx.x % p.n_proj;
  const int grp = blockIdx.x / p.n_proj;
  const int H = p.H;
  const int my_tiles = (grp < p.n_tiles) ? (p.n_tiles - 1 - grp) / p.groups + 1 : 0;
  pdl_launch_dependents();
  if (my_tiles == 0) {
    pdl_wait();
    return;
  }

  if (threadIdx.x == 0) {
    mbar_init(w_full, 1);
    for (int i = 0; i < NST; ++i) {
      mbar_init(x_full + i, 1);
      mbar_init(x_empty + i, 1);
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
  // set-up done: from here on global memory that the previous kernel writes
  pdl_wait();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx wc{p.err, abort_flag, p.timeout_ns};

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tm_x);
      mbar_arrive_expect_tx(w_full, Cfg::W_B);
      for (int kc = 0; kc < KC; ++kc)
        for (int na = 0; na < KC; ++na) {
          // each branch names its own kernel parameter, so the tensor map is
          // always read from parameter space
          void* dst = sw + (kc * KC + na) * Cfg::W_BOX;
          switch (proj) {
            case 0: tma_load_2d(dst, &tm_w0, w_full, na * 64, kc * 64); break;
            case 1: tma_load_2d(dst, &tm_w1, w_full, na * 64, kc * 64); break;
            case 2: tma_load_2d(dst, &tm_w2, w_full, na * 64, kc * 64); break;
            default: tma_load_2d(dst, &tm_w3, w_full, na * 64, kc * 64); break;
          }
        }
      int issued = 0;
      for (int i = 0; i < my_tiles; ++i) {
        const int tile = grp + i * p.groups;
        const int b = tile / p.tiles_per_b;
        const int n0 = (tile % p.tiles_per_b) * kProjTile;
        bool ok = true;
        for (int kc = 0; kc < KC; ++kc) {
          const int x = i * KC + kc, st = x % NST;
          if (!mbar_wait(x_empty + st, ((x / NST) & 1) ^ 1, wc)) { ok = false; break; }
          mbar_arrive_expect_tx(x_full + st, Cfg::X_B);
          tma_load_3d(sx + st * Cfg::X_B, &tm_x, x_full + st, kc * 64, n0, b);
          issued = x + 1;
        }
        if (!ok) break;
      }
      for (int x = max(0, issued - NST); x < issued; ++x)
        mbar_wait_drain(x_full + (x % NST), (x / NST) & 1, p.timeout_ns);
      mbar_wait_drain(w_full, 0, p.timeout_ns);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, C, false, true);
      const uint32_t sw_a = smem_u32(sw), sx_a = smem_u32(sx);
      bool ok = mbar_wait(w_full, 0, wc);
      for (int i = 0; ok && i < my_tiles; ++i) {
        const int ab = i & 1;
        if (i >= 2 && !mbar_wait(acc_free + ab, ((i >> 1) - 1) & 1, wc)) { ok = false; break; }
        tc_fence_after();
        for (int kc = 0; kc < KC; ++kc) {
          const int x = i * KC + kc, st = x % NST;
          if (!mbar_wait(x_full + st, (x / NST) & 1, wc)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            // A: X chunk, K-major SW128, k-step = 16 columns = 32 bytes inside the atom
            const uint64_t adesc = umma_desc(sx_a + st * Cfg::X_B + ks * 32, 16, 1024, LAYOUT_SW128);
            // B: W_p rows [kc*64 + 16ks, +16), MN-major SW128; N-atoms (64 cols) are W_BOX apart
            const uint64_t bdesc =
                umma_desc(sw_a + kc * KC * Cfg::W_BOX + ks * 16 * 128, Cfg::W_BOX, 1024, LAYOUT_SW128);
            umma_ss(tmem + ab * C, adesc, bdesc, idesc, (kc > 0 || ks > 0) ? 1u : 0u);
          }
          umma_commit(x_empty + st);
        }
        if (!ok) break;
        umma_commit(acc_full + ab);
      }
      umma_commit(mma_done);
      mbar_wait_drain(mma_done, 0, p.timeout_ns);
    }
  } else {
    const int wq = warp & 3;
    const int r = wq * 32 + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    uint16_t* out = proj == 0 ? p.out[0] : proj == 1 ? p.out[1] : proj == 2 ? p.out[2] : p.out[3];
    float* knorm = proj == 0 ? p.knorm[0] : proj == 1 ? p.knorm[1] : proj == 2 ? p.knorm[2] : p.knorm[3];
    for (int i = 0; i < my_tiles; ++i) {
      const int ab = i & 1;
      const int tile = grp + i * p.groups;
      const int b = tile / p.tiles_per_b;
      const int n0 = (tile % p.tiles_per_b) * kProjTile;
      const int n = n0 + r;
      if (!mbar_wait_warp(acc_full + ab, (i >> 1) & 1, wc)) break;
      tc_fence_after();
      // G heads per TMEM read (one wait per G heads; G * D columns)
      constexpr int G = D == 16 ? FLARE_PROJ_EPI_HEADS : (FLARE_PROJ_EPI_HEADS + 1) / 2;
      for (int h0 = 0; h0 < H; h0 += G) {
        uint32_t v[G][D];
#pragma unroll
        for (int j = 0; j < G; ++j)
          if (h0 + j < H) tmem_ld_cols<D>(lane_base + ab * C + (h0 + j) * D, v[j]);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < G; ++j) {
          const int hh = h0 + j;
          if (hh >= H) break;
          uint32_t pk[D / 2];
          float nrm = 0.f;
#pragma unroll
          for (int k = 0; k < D / 2; ++k) {
            pk[k] = pack_bf16x2(__uint_as_float(v[j][2 * k]), __uint_as_float(v[j][2 * k + 1]));
            const float a = bf16_lo(pk[k]), bb = bf16_hi(pk[k]);
            nrm = fmaf(a, a, fmaf(bb, bb, nrm));
          }
          if (n < p.N) {
            const size_t row = p.token_major ? (static_cast<size_t>(b) * p.N + n) * p.C + hh * D
                                             : ((static_cast<size_t>(b) * H + hh) * p.N + n) * D;
            uint4* dst = reinterpret_cast<uint4*>(out + row);
#pragma unroll
            for (int u = 0; u < D / 8; ++u)
              dst[u] = make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
          } else {
            nrm = 0.f;
          }
          if (knorm != nullptr) {
            const float gm = warp_max_nonneg(sqrtf(nrm));
            const int gi = n0 / kNormGroup + wq;
            if (lane == 0 && gi < p.n_groups32)
              knorm[(static_cast<size_t>(b) * H + hh) * p.n_groups32 + gi] = gm;
          }
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

template <int C, int D>
cudaError_t launch_project_cd(const CUtensorMap& tm_x, const CUtensorMap (&tm_w)[4], const ProjParams& p,
                              cudaStream_t s, bool pdl) {
  const size_t smem = project_smem_bytes(C);
  cudaError_t e = cudaFuncSetAttribute(project_kernel<C, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  LaunchCfg lc(dim3(p.n_proj * p.groups), dim3(192), smem, s, pdl);
  return cudaLaunchKernelEx(&lc.cfg, project_kernel<C, D>, tm_x, tm_w[0], tm_w[1], tm_w[2], tm_w[3], p);
}

template <int C>
cudaError_t launch_project_c(const CUtensorMap& tm_x, const CUtensorMap (&tm_w)[4], const ProjParams& p,
                             cudaStream_t s, bool pdl) {
  return p.D == 16 ? launch_project_cd<C, 16>(tm_x, tm_w, p, s, pdl) : launch_project_cd<C, 32>(tm_x, tm_w, p, s, pdl);
}

}  // namespace

size_t project_smem_bytes(int C) {
  size_t need = 0;
  if (C == 64) need = ProjCfg<64>::BYTES;
  else if (C == 128) need = ProjCfg<128>::BYTES;
  else need = ProjCfg<256>::BYTES;
  need += 1024;
  // at most two co-resident CTAs per SM (TMEM: 2*C columns each)
  return need > 90 * 1024 ? need : 90 * 1024;
}

cudaError_t launch_project(const CUtensorMap& tm_x, const CUtensorMap (&tm_w)[4], const ProjParams& p,
                           cudaStream_t s, bool pdl) {
  switch (p.C) {
    case 64: return launch_project_c<64>(tm_x, tm_w, p, s, pdl);
    case 128: return launch_project_c<128>(tm_x, tm_w, p, s, pdl);
    case 256: return launch_project_c<256>(tm_x, tm_w, p, s, pdl);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace flare
