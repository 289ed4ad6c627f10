// Small kernels around the encoder:
//  - merge_kernel: combines the per-split partial softmax sums of the encoder
//    with the log-sum-exp rule of the FLARE++ paper (arXiv 2608.11519,
//    section "Multi-GPU context parallelism", eq. 14), used here across the
//    CTAs of one GPU instead of across ranks.  Splits are visited in
//    ascending order, so the result is bitwise reproducible.  A row whose
//    fast-path sums lost mass to underflow is recomputed exactly (two-pass
//    softmax in fp32 over all valid tokens) by the warp that owns it; across
//    shards (context parallelism) no rank holds all tokens, so each rank
//    computes the exact partial sums of its own tokens for such rows
//    (cp_exact_kernel), the ranks exchange them, and the merge combines
//    those with the same log-sum-exp rule.
//  - knorm_kernel: largest key norm of every 32-token group (keys given by
//    the caller, FLARE path); the encoder's softmax shift bound.
//  - wait_selftest_kernel: exercises the bounded-wait error path.
#include "ptx.cuh"

namespace flare {
namespace {

// Exact partial sums of one encoder row over the tokens n < L of kh / vh,
// fp32, two passes: mx = max_n <q, k_n> * c (log2 units), den = sum_n
// 2^(<q, k_n> c - mx) and acc = the same sum of v_n[d] (den >= 1: the
// largest term is 1, so nothing underflows that matters).  lane = (group,
// d): the 32 / D groups take the tokens n = group, group + 32 / D, ...; a dot
// product is a butterfly over the D lanes of a group.  Every reduction has a
// fixed order.  acc is this lane's d; L <= 0 gives (-inf, 0, 0).
struct ExactPartial {
  float mx, den, acc;
};
template <int D>
__device__ ExactPartial exact_partial(const MergeParams& p, const uint16_t* qrow, const uint16_t* kh,
                                      const uint16_t* vh, int L, int lane) {
  if (L <= 0) return {-INFINITY, 0.f, 0.f};
  constexpr int NG = 32 / D;
  const int d = lane % D, grp = lane / D;
  const float qd = __uint_as_float(static_cast<uint32_t>(qrow[d]) << 16);
  auto score = [&](int n) {  // <q, k_n> * c, the same in every lane of the group
    float t = qd * __uint_as_float(static_cast<uint32_t>(kh[static_cast<size_t>(n) * D + d]) << 16);
#pragma unroll
    for (int o = 1; o < D; o <<= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    return t * p.c;
  };
  // every lane of the warp runs the same number of iterations (the shuffles
  // need the whole warp); tokens past L are skipped arithmetically
  const int iters = (L + NG - 1) / NG;
  float mx = -INFINITY;
  for (int it = 0; it < iters; ++it) {
    const int n = it * NG + grp;
    const float sc = score(min(n, L - 1));
    if (n < L) mx = fmaxf(mx, sc);
  }
  mx = warp_max(mx);
  float acc = 0.f, den = 0.f;
  for (int it = 0; it < iters; ++it) {
    const int n = it * NG + grp;
    const float sc = score(min(n, L - 1));
    if (n < L) {
      const float e = exp2f(sc - mx);
      den += e;
      acc = fmaf(e, __uint_as_float(static_cast<uint32_t>(vh[static_cast<size_t>(n) * D + d]) << 16), acc);
    }
  }
#pragma unroll
  for (int o = D; o < 32; o <<= 1) {
    acc += __shfl_xor_sync(0xffffffffu, acc, o);
    den += __shfl_xor_sync(0xffffffffu, den, o);
  }
  return {mx, den, acc};
}

// What the split partials of one row (b, h, m) say, identically in every
// lane: G = log2 of the row's total weight, max over the splits of all
// shards of U + log2 l (-inf if every sum is zero); has_tokens: some split
// holds a valid token; needs_exact: the fast-path sums may have lost more
// than 2^-27 of the row's mass to flushed exponentials (bound: every token
// of a split at 2^(U - 126)), or lost all of it.  The merge and the
// context-parallel exact pass decide with this one function, so they agree.
struct RowStats {
  float G;
  bool has_tokens, needs_exact;
};
template <int D>
__device__ RowStats row_stats(const MergeParams& p, int bh, int m, int b, int lane) {
  const int S = p.n_splits, R = p.n_ranks;
  const size_t stride = static_cast<size_t>(p.M) * (D + 2);
  bool bad = false;
  float G = -INFINITY, lost = -INFINITY;
  bool any = false;
  // Lanes take the splits j = lane, lane + 32, ... (j = r * S + s); the
  // butterfly reductions below have a fixed order (bitwise reproducible).
  for (int j = lane; j < R * S; j += 32) {
    const int r = j / S, s = j - r * S;
    const int Lr = shard_valid_len(p.lengths, b, p.N, r * p.N, R * p.N, &bad);
    const int ntv = (Lr + enc_tile(D) - 1) / enc_tile(D);
    const int t0 = s * p.tiles_per_split, t1 = min(t0 + p.tiles_per_split, ntv);
    const int nt = max(0, t1 - t0);
    if (nt == 0) continue;
    any = true;
    const float2 ul = *reinterpret_cast<const float2*>(p.part + r * p.rank_stride +
                                                      (static_cast<size_t>(bh) * S + s) * stride +
                                                      static_cast<size_t>(m) * (D + 2));
    if (ul.y > 0.f) G = fmaxf(G, ul.x + log2f(ul.y));
    lost = fmaxf(lost, ul.x - 126.f + log2f(static_cast<float>(nt * enc_tile(D))));
  }
  G = warp_max(G);
  lost = warp_max(lost);
  any = __any_sync(0xffffffffu, any);
  const bool needs = any && (!(G > -INFINITY) || (lost + log2f(static_cast<float>(R * S)) - G > -27.f));
  return {G, any, needs};
}

// From this many (shard, split) partials per row on, the merge gives every
// lane whole splits (one round of loads) instead of one value of d.
constexpr int kMergeLanesOverSplits = 12;

template <int D>
__global__ void __launch_bounds__(256) merge_kernel(const MergeParams p) {
  pdl_launch_dependents();
  pdl_wait();
  const int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= p.B * p.H * p.M) return;
  const int bh = row / p.M, m = row % p.M;
  const int b = bh / p.H, h = bh % p.H;
  const int S = p.n_splits, R = p.n_ranks;
  const size_t stride = static_cast<size_t>(p.M) * (D + 2);
  // partials of split s of shard r: (U, l, O[D]) of this row
  auto part_of = [&](int r, int s) {
    return p.part + r * p.rank_stride + (static_cast<size_t>(bh) * S + s) * stride + static_cast<size_t>(m) * (D + 2);
  };
  // token tiles of split s of shard r that hold valid tokens
  bool bad = false;
  auto split_tiles = [&](int r, int s) {
    const int Lr = shard_valid_len(p.lengths, b, p.N, r * p.N, R * p.N, &bad);
    const int ntv = (Lr + enc_tile(D) - 1) / enc_tile(D);
    const int t0 = s * p.tiles_per_split, t1 = min(t0 + p.tiles_per_split, ntv);
    return max(0, t1 - t0);
  };
  const RowStats rs = row_stats<D>(p, bh, m, b, lane);
  const float G = rs.G;
  // lane = (group, d): the 32 / D groups take the splits (or shards) j =
  // group, group + 32 / D, ... in ascending order; one value of d per lane
  // keeps the registers (and so the occupancy) independent of D
  constexpr int NG = 32 / D;
  const int d = lane % D, grp = lane / D;
  float z = 0.f;
  float lse = -INFINITY;  // log2 of the row's total weight, for lse_out
  const bool can_exact = R == 1 && p.allow_exact;
  if (!rs.has_tokens) {
    z = 0.f;
  } else if (rs.needs_exact && can_exact) {
    const int g = p.q_per_batch ? bh : h;
    const int L = shard_valid_len(p.lengths, b, p.N, 0, p.N, &bad);
    const ExactPartial e =
        exact_partial<D>(p, p.q + (static_cast<size_t>(g) * p.M + m) * D, p.k + static_cast<size_t>(bh) * p.N * D,
                         p.v + static_cast<size_t>(bh) * p.N * D, L, lane);
    z = L > 0 ? e.acc / e.den : 0.f;
    lse = e.mx + log2f(e.den);
  } else if (rs.needs_exact && p.fix != nullptr) {
    // every shard's exact partial sums of this row: (mx, den, acc[D]), rank-major
    const float* fr = p.fix + static_cast<size_t>(row) * (D + 2);
    float G2 = -INFINITY;
    for (int r = lane; r < R; r += 32) {
      const float2 md = *reinterpret_cast<const float2*>(fr + r * p.fix_rank_stride);
      if (md.y > 0.f) G2 = fmaxf(G2, md.x + log2f(md.y));
    }
    G2 = warp_max(G2);
    float num = 0.f, den = 0.f;
    for (int r = grp; r < R; r += NG) {
      const float* e = fr + r * p.fix_rank_stride;
      if (!(e[1] > 0.f)) continue;
      const float w = exp2f(e[0] - G2);
      den = fmaf(w, e[1], den);
      num = fmaf(w, e[2 + d], num);
    }
#pragma unroll
    for (int o = D; o < 32; o <<= 1) {
      num += __shfl_xor_sync(0xffffffffu, num, o);
      den += __shfl_xor_sync(0xffffffffu, den, o);
    }
    z = num / den;
    lse = G2 + log2f(den);
  } else if (G > -INFINITY && R * S < kMergeLanesOverSplits) {
    // few splits: the 32 / D lane groups take the splits j = group,
    // group + 32 / D, ..., each lane one value of d
    float num = 0.f, den = 0.f;
#pragma unroll 4
    for (int j = grp; j < R * S; j += NG) {
      const int r = j / S, s = j - r * S;
      if (split_tiles(r, s) == 0) continue;
      const float* e = part_of(r, s);  // (U, l, O[D])
      const float2 ul = *reinterpret_cast<const float2*>(e);
      if (!(ul.y > 0.f)) continue;
      const float w = exp2f(ul.x - G);
      den = fmaf(w, ul.y, den);
      num = fmaf(w, e[2 + d], num);
    }
#pragma unroll
    for (int o = D; o < 32; o <<= 1) {  // combine the groups (commutative adds: same bits in every lane)
      num += __shfl_xor_sync(0xffffffffu, num, o);
      den += __shfl_xor_sync(0xffffffffu, den, o);
    }
    z = num / den;
    lse = G + log2f(den);
    if (rs.needs_exact && lane == 0) atomicOr(p.err, FLARE_DEV_UNDERFLOW);
  } else {
    if (G > -INFINITY) {
      // many splits: every lane takes whole splits j = lane, lane + 32, ...
      // (one row of D + 2 floats each, all loads of the warp in flight at
      // once), then a butterfly over the lanes; each step adds two lanes'
      // values, a commutative operation, so every lane ends with the same bits
      float num[D], den = 0.f;
#pragma unroll
      for (int k = 0; k < D; ++k) num[k] = 0.f;
      for (int j = lane; j < R * S; j += 32) {
        const int r = j / S, s = j - r * S;
        if (split_tiles(r, s) == 0) continue;
        const float2* e = reinterpret_cast<const float2*>(part_of(r, s));  // (U, l), then O[D] as pairs
        const float2 ul = e[0];
        if (!(ul.y > 0.f)) continue;
        const float w = exp2f(ul.x - G);
        den = fmaf(w, ul.y, den);
#pragma unroll
        for (int k = 0; k < D / 2; ++k) {
          const float2 o = e[1 + k];
          num[2 * k] = fmaf(w, o.x, num[2 * k]);
          num[2 * k + 1] = fmaf(w, o.y, num[2 * k + 1]);
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        den += __shfl_xor_sync(0xffffffffu, den, o);
#pragma unroll
        for (int k = 0; k < D; ++k) num[k] += __shfl_xor_sync(0xffffffffu, num[k], o);
      }
      float mine = 0.f;
#pragma unroll
      for (int k = 0; k < D; ++k)
        if (k == d) mine = num[k];
      z = mine / den;
      lse = G + log2f(den);
    }
    // a row that needed the exact recomputation, with no exact partials of
    // the other shards at hand, is reported instead
    if (rs.needs_exact && lane == 0) atomicOr(p.err, FLARE_DEV_UNDERFLOW);
  }
  if (p.lse_out != nullptr && lane == 0) p.lse_out[row] = lse;
  if (lane < D) {
    const size_t o = static_cast<size_t>(row) * D + lane;
    p.out_f32[o] = z;
    p.out_bf16[o] = static_cast<uint16_t>(pack_bf16x2(z, 0.f) & 0xFFFFu);
  }
}

// Context parallelism: for every row that the merge of the gathered split
// partials will find in need of the exact recomputation (row_stats), this
// rank's exact partial sums over its own valid tokens; other rows get
// (-inf, 0, 0).  p.N is the shard's token count, p.q / p.k / p.v the
// shard's queries, keys and values; out: [B*H*M][D+2].
template <int D>
__global__ void __launch_bounds__(256) cp_exact_kernel(const MergeParams p, int rank, float* out) {
  pdl_wait();
  const int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= p.B * p.H * p.M) return;
  const int bh = row / p.M, m = row % p.M;
  const int b = bh / p.H, h = bh % p.H;
  const RowStats rs = row_stats<D>(p, bh, m, b, lane);
  ExactPartial e{-INFINITY, 0.f, 0.f};
  if (rs.needs_exact) {
    bool bad = false;
    const int L = shard_valid_len(p.lengths, b, p.N, rank * p.N, p.n_ranks * p.N, &bad);
    const int g = p.q_per_batch ? bh : h;
    e = exact_partial<D>(p, p.q + (static_cast<size_t>(g) * p.M + m) * D, p.k + static_cast<size_t>(bh) * p.N * D,
                         p.v + static_cast<size_t>(bh) * p.N * D, L, lane);
  }
  float* o = out + static_cast<size_t>(row) * (D + 2);
  if (lane == 0) {
    o[0] = e.mx;
    o[1] = e.den;
  }
  if (lane < D) o[2 + lane] = e.acc;
}

template <int D>
__global__ void __launch_bounds__(256) knorm_kernel(const KnormParams p) {
  pdl_launch_dependents();
  pdl_wait();
  const long grp = (static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (grp >= static_cast<long>(p.BH) * p.n_groups32) return;
  const int bh = static_cast<int>(grp / p.n_groups32), gi = static_cast<int>(grp % p.n_groups32);
  const int n = gi * kNormGroup + lane;
  float s = 0.f;
  if (n < p.N) {
    const uint4* row = reinterpret_cast<const uint4*>(p.k + (static_cast<size_t>(bh) * p.N + n) * D);
#pragma unroll
    for (int u = 0; u < D / 8; ++u) {
      const uint4 v = row[u];
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const float a = bf16_lo(w[t]), b = bf16_hi(w[t]);
        s = fmaf(a, a, fmaf(b, b, s));
      }
    }
  }
  const float nm = warp_max(sqrtf(s));
  if (lane == 0) p.knorm[grp] = nm;
}

__global__ void wait_selftest_kernel(uint32_t* err, unsigned long long timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // nothing ever arrives on `bar`: the wait runs out and records the error
    const WaitCtx w{err, &abort_flag, timeout_ns};
    mbar_wait(&bar, 0, w);
  }
}

__global__ void __launch_bounds__(256) to_f16_kernel(const ToF16Params p) {
  const long i = 2 * (static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x);
  if (i >= p.n) return;
  const float2 f = *reinterpret_cast<const float2*>(p.src + i);
  *reinterpret_cast<uint32_t*>(p.dst + i) = pack_f16x2(f.x, f.y);
}

}  // namespace

cudaError_t launch_to_f16(const ToF16Params& p, cudaStream_t s) {
  const long pairs = p.n / 2;
  to_f16_kernel<<<static_cast<unsigned>((pairs + 255) / 256), 256, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_merge(const MergeParams& p, cudaStream_t s, bool pdl) {
  const long rows = static_cast<long>(p.B) * p.H * p.M;
  LaunchCfg lc(dim3(static_cast<unsigned>((rows * 32 + 255) / 256)), dim3(256), 0, s, pdl);
  return p.D == 16 ? cudaLaunchKernelEx(&lc.cfg, merge_kernel<16>, p) : cudaLaunchKernelEx(&lc.cfg, merge_kernel<32>, p);
}

cudaError_t launch_cp_exact(const MergeParams& p, int rank, float* out, cudaStream_t s) {
  const long rows = static_cast<long>(p.B) * p.H * p.M;
  const dim3 grid(static_cast<unsigned>((rows * 32 + 255) / 256));
  if (p.D == 16) cp_exact_kernel<16><<<grid, 256, 0, s>>>(p, rank, out);
  else cp_exact_kernel<32><<<grid, 256, 0, s>>>(p, rank, out);
  return cudaGetLastError();
}

cudaError_t launch_knorm(const KnormParams& p, cudaStream_t s) {
  const long groups = static_cast<long>(p.BH) * p.n_groups32;
  const dim3 grid(static_cast<unsigned>((groups * 32 + 255) / 256));
  if (p.D == 16) knorm_kernel<16><<<grid, 256, 0, s>>>(p);
  else knorm_kernel<32><<<grid, 256, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_wait_selftest(uint32_t* err, unsigned long long timeout_ns, cudaStream_t s) {
  wait_selftest_kernel<<<1, 32, 0, s>>>(err, timeout_ns);
  return cudaGetLastError();
}

}  // namespace flare
