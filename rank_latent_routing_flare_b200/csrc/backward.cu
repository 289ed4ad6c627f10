// Gradient kernels of the FLARE / FLARE++ mixer, fp32 on the CUDA cores.
//
// Every step of the mixer is one SDPA call (FLARE++ paper, arXiv
// 2608.11519, section "FLARE++: dynamic token routing", eq. 8, 10, 11); the
// paper's own backward equations (eq. 13-40) are named but not printed on
// the pages, so these kernels compute the SDPA backward of each call:
//   O = softmax_rows(s Qa Ka^T) Va, upstream dO, weights P:
//   dVa = P^T dO,  dS = P (dO Va^T - delta),  delta_r = <dO_r, O_r>,
//   dQa = s dS Ka,  dKa = s dS^T Qa.
// The softmax weights are recomputed from row log-normalisers (log2 units:
// scores t = scale * log2(e) * <q, k>, weights 2^(t - L)), which the
// recompute kernels here produce in fp32: the encoder's per latent row
// (latent-parallel pass, split over tokens, merged in a fixed order) and the
// decoder's per token (token-parallel pass over all latents).
//
// Kernels:
//   lat_kernel<kLatForward>  encoder recompute partials (max, sum, sum w v)
//   lat_merge_kernel         Z and the encoder row log-normalisers
//   tok_kernel<kTokStats>    decoder per-token log-normaliser and delta
//   lat_kernel<kLatDecoder>  dZ = P^T dY and the decoder's dQ (per split)
//   lat_sum_kernel           fixed-order sums of split partials (+ gamma)
//   tok_kernel<kTokFull>     dK (decoder + encoder) and dV
//   lat_kernel<kLatEncoder>  the encoder's dQ (per split)
//   tok_kernel<kTokEncoder>  dK, dV of the query synthesis
//   dx_kernel / dw_kernel / dw_reduce_kernel   projection gradients
// Every reduction has a fixed order: the results are bitwise reproducible.
#include "bwd_internal.h"
#include "flare_internal.h"
#include "ptx.cuh"

namespace flare {
namespace {

constexpr int kDH = 16;  // feature dimensions held per thread
constexpr unsigned kAll = 0xffffffffu;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ float bf(uint16_t x) { return __uint_as_float(static_cast<uint32_t>(x) << 16); }

__device__ __forceinline__ uint16_t to_bf16(float x) { return static_cast<uint16_t>(pack_bf16x2(x, 0.f) & 0xFFFFu); }

// Sum over the TPR threads of one row (adjacent lanes).
template <int TPR>
__device__ __forceinline__ float row_sum(float x) {
  if (TPR == 2) x += __shfl_xor_sync(kAll, x, 1);
  return x;
}

__device__ __forceinline__ float dot16(const float (&a)[kDH], const float (&b)[kDH]) {
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < kDH; ++i) s = fmaf(a[i], b[i], s);
  return s;
}

// 16 floats from shared memory (16-byte aligned).
__device__ __forceinline__ void lds16(float (&r)[kDH], const float* p) {
  const float4* q = reinterpret_cast<const float4*>(p);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float4 t = q[i];
    r[4 * i] = t.x;
    r[4 * i + 1] = t.y;
    r[4 * i + 2] = t.z;
    r[4 * i + 3] = t.w;
  }
}

// 16 bf16 values from global memory (32-byte aligned), widened.
__device__ __forceinline__ void ldg16_bf16(float (&r)[kDH], const uint16_t* p) {
  const uint4* q = reinterpret_cast<const uint4*>(p);
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const uint4 t = q[i];
    const uint32_t w[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      r[8 * i + 2 * j] = bf16_lo(w[j]);
      r[8 * i + 2 * j + 1] = bf16_hi(w[j]);
    }
  }
}

// ---------------------------------------------------------------------------
// Latent-parallel pass: a thread owns one latent row m (D = 32: two threads,
// 16 dimensions each) and walks the valid tokens of its split in tiles that
// the CTA stages in shared memory as fp32.
// ---------------------------------------------------------------------------
template <int D, int MODE>
__global__ void __launch_bounds__(256) lat_kernel(const LatParams p) {
  constexpr int TPR = D / kDH;
  constexpr int T = kBwdTokTile;
  __shared__ __align__(16) float sK[T * D];
  __shared__ __align__(16) float sX[T * D];  // V (forward, encoder) or dY (decoder)
  __shared__ float sL[T], sDl[T];

  const int tid = threadIdx.x;
  const int row = tid / TPR, part = tid % TPR;
  const int split = blockIdx.x, bh = blockIdx.z;
  const int m = blockIdx.y * p.rows_per_block + row;
  const bool active = m < p.M;
  const int b = bh / p.H, h = bh % p.H;
  const int g = p.q_per_batch ? bh : h;
  bool bad = false;
  const int L = shard_valid_len(p.lengths, b, p.N, 0, p.N, &bad);
  if (bad && tid == 0 && split == 0 && blockIdx.y == 0) atomicOr(p.err, FLARE_DEV_BAD_LENGTH);
  const int ntv = (L + T - 1) / T;
  const int t_begin = split * p.tiles_per_split;
  const int t_end = min(t_begin + p.tiles_per_split, ntv);

  // this thread's query (log2-scaled) and row vector; inactive rows compute
  // on zeros (every thread takes part in the shuffles) and write nothing
  float qv[kDH], zv[kDH], accA[kDH], accB[kDH];
  const size_t qoff = (static_cast<size_t>(g) * p.M + (active ? m : 0)) * D + part * kDH;
  const size_t roff = (static_cast<size_t>(bh) * p.M + (active ? m : 0)) * D + part * kDH;
#pragma unroll
  for (int i = 0; i < kDH; ++i) {
    qv[i] = active ? p.c * p.q[qoff + i] : 0.f;
    zv[i] = (MODE != kLatForward && active) ? p.zrow[roff + i] : 0.f;
    accA[i] = 0.f;
    accB[i] = 0.f;
  }
  float mx = -INFINITY, l = 0.f, lrow = 0.f, grow = 0.f;
  if (MODE == kLatEncoder && active) {
    lrow = p.lrow[static_cast<size_t>(bh) * p.M + m];
    grow = p.grow[static_cast<size_t>(bh) * p.M + m];
  }

  const uint16_t* kh = p.k + static_cast<size_t>(bh) * p.N * D;
  const uint16_t* xh = (MODE == kLatDecoder ? p.dy : p.v) + static_cast<size_t>(bh) * p.N * D;
  for (int t = t_begin; t < t_end; ++t) {
    const int n0 = t * T;
    const int nt = min(T, L - n0);
    __syncthreads();  // the previous tile has been consumed
    const uint32_t* k32 = reinterpret_cast<const uint32_t*>(kh + static_cast<size_t>(n0) * D);
    const uint32_t* x32 = reinterpret_cast<const uint32_t*>(xh + static_cast<size_t>(n0) * D);
    for (int i = tid; i < T * D / 2; i += blockDim.x) {
      const bool in = (2 * i) / D < nt;
      const uint32_t wk = in ? k32[i] : 0u, wx = in ? x32[i] : 0u;
      reinterpret_cast<float2*>(sK)[i] = make_float2(bf16_lo(wk), bf16_hi(wk));
      reinterpret_cast<float2*>(sX)[i] = make_float2(bf16_lo(wx), bf16_hi(wx));
    }
    if (MODE == kLatDecoder) {
      for (int j = tid; j < T; j += blockDim.x) {
        const size_t o = static_cast<size_t>(bh) * p.N + n0 + j;
        sL[j] = j < nt ? p.ltok[o] : 0.f;
        sDl[j] = j < nt ? p.dtok[o] : 0.f;
      }
    }
    __syncthreads();
    for (int j = 0; j < nt; ++j) {
      float kj[kDH], xj[kDH];
      lds16(kj, sK + j * D + part * kDH);
      lds16(xj, sX + j * D + part * kDH);
      const float s = row_sum<TPR>(dot16(qv, kj));
      if (MODE == kLatForward) {
        // online softmax in log2 units; both threads of a row see the same s
        if (s > mx) {
          const float r = ex2_mufu(mx - s);
          l = fmaf(l, r, 1.f);
#pragma unroll
          for (int i = 0; i < kDH; ++i) accA[i] = fmaf(accA[i], r, xj[i]);
          mx = s;
        } else {
          const float w = ex2_mufu(s - mx);
          l += w;
#pragma unroll
          for (int i = 0; i < kDH; ++i) accA[i] = fmaf(w, xj[i], accA[i]);
        }
      } else if (MODE == kLatDecoder) {
        // P[n][m] = 2^(t - L_n); dS = P (<dY_n, Z_m> - delta_n)
        const float w = ex2_mufu(s - sL[j]);
        const float ds = w * (row_sum<TPR>(dot16(zv, xj)) - sDl[j]);
#pragma unroll
        for (int i = 0; i < kDH; ++i) {
          accA[i] = fmaf(w, xj[i], accA[i]);
          accB[i] = fmaf(ds, kj[i], accB[i]);
        }
      } else {
        // A[m][n] = 2^(t - L_m); dS = A (<dZ_m, V_n> - gamma_m)
        const float w = ex2_mufu(s - lrow);
        const float ds = w * (row_sum<TPR>(dot16(zv, xj)) - grow);
#pragma unroll
        for (int i = 0; i < kDH; ++i) accB[i] = fmaf(ds, kj[i], accB[i]);
      }
    }
  }
  if (!active) return;
  const size_t base = (static_cast<size_t>(bh) * p.n_splits + split) * p.M + m;
  if (MODE == kLatForward) {
    float* o = p.part_a + base * (D + 2);
    if (part == 0) {
      o[0] = mx;
      o[1] = l;
    }
#pragma unroll
    for (int i = 0; i < kDH; ++i) o[2 + part * kDH + i] = accA[i];
  } else {
    if (MODE == kLatDecoder) {
      float4* oa = reinterpret_cast<float4*>(p.part_a + base * D + part * kDH);
#pragma unroll
      for (int i = 0; i < 4; ++i) oa[i] = make_float4(accA[4 * i], accA[4 * i + 1], accA[4 * i + 2], accA[4 * i + 3]);
    }
    float4* ob = reinterpret_cast<float4*>(p.part_b + base * D + part * kDH);
#pragma unroll
    for (int i = 0; i < 4; ++i) ob[i] = make_float4(accB[4 * i], accB[4 * i + 1], accB[4 * i + 2], accB[4 * i + 3]);
  }
}

// Encoder recompute: merge of the split partials of one latent row, in
// ascending split order: Z[m] and L_m = log2 sum_n 2^(t_mn).
template <int D>
__global__ void __launch_bounds__(256) lat_merge_kernel(const LatMergeParams p) {
  const long r = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (r >= static_cast<long>(p.BH) * p.M) return;
  const long bh = r / p.M, m = r % p.M;
  const size_t sstride = static_cast<size_t>(p.M) * (D + 2);
  const float* base = p.part + (static_cast<size_t>(bh) * p.S * p.M + m) * (D + 2);
  float G = -INFINITY;
  for (int s = 0; s < p.S; ++s) {
    const float* e = base + s * sstride;
    if (e[1] > 0.f) G = fmaxf(G, e[0]);
  }
  float den = 0.f, acc[D];
#pragma unroll
  for (int d = 0; d < D; ++d) acc[d] = 0.f;
  for (int s = 0; s < p.S; ++s) {
    const float* e = base + s * sstride;
    if (!(e[1] > 0.f)) continue;
    const float w = ex2_mufu(e[0] - G);
    den = fmaf(w, e[1], den);
#pragma unroll
    for (int d = 0; d < D; ++d) acc[d] = fmaf(w, e[2 + d], acc[d]);
  }
#pragma unroll
  for (int d = 0; d < D; ++d) p.z[r * D + d] = acc[d] / den;
  p.lse[r] = G + __log2f(den);
}

// Fixed-order sum of split partials (and, for shared queries, of the batch):
// out = mult * sum; gamma = <out, zref> per row when zref is given.
template <int D>
__global__ void __launch_bounds__(256) lat_sum_kernel(const LatSumParams p) {
  const int rows = (p.fold_batch ? p.H : p.B * p.H) * p.M;
  const int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= rows) return;
  const int grp = r / p.M, m = r % p.M;
  float acc[D];
#pragma unroll
  for (int d = 0; d < D; ++d) acc[d] = 0.f;
  const int nb = p.fold_batch ? p.B : 1;
  for (int bi = 0; bi < nb; ++bi) {
    const int bh = p.fold_batch ? bi * p.H + grp : grp;
    for (int pi = 0; pi < 2; ++pi) {
      const float* part = pi == 0 ? p.part0 : p.part1;
      if (part == nullptr) continue;
      for (int s = 0; s < p.S; ++s) {
        const float4* e = reinterpret_cast<const float4*>(part + ((static_cast<size_t>(bh) * p.S + s) * p.M + m) * D);
#pragma unroll
        for (int u = 0; u < D / 4; ++u) {
          const float4 t = e[u];
          acc[4 * u] += t.x;
          acc[4 * u + 1] += t.y;
          acc[4 * u + 2] += t.z;
          acc[4 * u + 3] += t.w;
        }
      }
    }
  }
  float gsum = 0.f;
#pragma unroll
  for (int d = 0; d < D; ++d) {
    acc[d] *= p.mult;
    p.out[static_cast<size_t>(r) * D + d] = acc[d];
    if (p.zref) gsum = fmaf(acc[d], p.zref[static_cast<size_t>(r) * D + d], gsum);
  }
  if (p.zref) p.gamma[r] = gsum;
}

// ---------------------------------------------------------------------------
// Token-parallel pass: a thread owns one token row (D = 32: two threads) and
// walks all latents in chunks that the CTA stages in shared memory.
// ---------------------------------------------------------------------------
template <int D, int MODE>
__global__ void __launch_bounds__(256) tok_kernel(const TokParams p) {
  constexpr int TPR = D / kDH;
  constexpr int MC = kBwdLatChunk;
  __shared__ __align__(16) float sQ[MC * D];   // log2-scaled queries
  __shared__ __align__(16) float sA[MC * D];   // Z (stats) or dZ
  __shared__ __align__(16) float sZ[MC * D];   // Z (full)
  __shared__ float sLm[MC], sG[MC];

  const int tid = threadIdx.x, row = tid / TPR, part = tid % TPR;
  const int bh = blockIdx.y, b = bh / p.H, h = bh % p.H;
  const int g = p.q_per_batch ? bh : h;
  const int n = blockIdx.x * kBwdTokBlock + row;
  bool bad = false;
  const int L = shard_valid_len(p.lengths, b, p.N, 0, p.N, &bad);
  const bool in_range = n < p.N;
  const bool valid = n < L;
  const size_t tok = static_cast<size_t>(bh) * p.N + (in_range ? n : 0);

  float kv[kDH], vv[kDH], dyv[kDH], accA[kDH], accB[kDH];
#pragma unroll
  for (int i = 0; i < kDH; ++i) {
    kv[i] = vv[i] = dyv[i] = 0.f;
    accA[i] = accB[i] = 0.f;
  }
  if (in_range) {
    ldg16_bf16(kv, p.k + tok * D + part * kDH);
    if (MODE != kTokStats) ldg16_bf16(vv, p.v + tok * D + part * kDH);
    if (MODE != kTokEncoder) ldg16_bf16(dyv, p.dy + tok * D + part * kDH);
  }
  float ln = 0.f, dl = 0.f;
  if (MODE == kTokFull && in_range) {
    ln = p.ltok[tok];
    dl = p.dtok[tok];
  }
  float mx = -INFINITY, l = 0.f;

  const float* qg = p.q + static_cast<size_t>(g) * p.M * D;
  const float* zb = p.z + static_cast<size_t>(bh) * p.M * D;
  const float* dzb = p.dz + static_cast<size_t>(bh) * p.M * D;
  for (int m0 = 0; m0 < p.M; m0 += MC) {
    const int mc = min(MC, p.M - m0);
    __syncthreads();  // the previous chunk has been consumed
    for (int i = tid; i < mc * D; i += blockDim.x) {
      sQ[i] = p.c * qg[static_cast<size_t>(m0) * D + i];
      if (MODE == kTokStats) {
        sA[i] = zb[static_cast<size_t>(m0) * D + i];
      } else {
        sA[i] = dzb[static_cast<size_t>(m0) * D + i];
        if (MODE == kTokFull) sZ[i] = zb[static_cast<size_t>(m0) * D + i];
      }
    }
    if (MODE != kTokStats) {
      for (int i = tid; i < mc; i += blockDim.x) {
        sLm[i] = p.lm[static_cast<size_t>(bh) * p.M + m0 + i];
        sG[i] = p.gam[static_cast<size_t>(bh) * p.M + m0 + i];
      }
    }
    __syncthreads();
    for (int j = 0; j < mc; ++j) {
      float qj[kDH], aj[kDH];
      lds16(qj, sQ + j * D + part * kDH);
      lds16(aj, sA + j * D + part * kDH);
      const float s = row_sum<TPR>(dot16(kv, qj));
      if (MODE == kTokStats) {
        if (s > mx) {
          const float r = ex2_mufu(mx - s);
          l = fmaf(l, r, 1.f);
#pragma unroll
          for (int i = 0; i < kDH; ++i) accA[i] = fmaf(accA[i], r, aj[i]);
          mx = s;
        } else {
          const float w = ex2_mufu(s - mx);
          l += w;
#pragma unroll
          for (int i = 0; i < kDH; ++i) accA[i] = fmaf(w, aj[i], accA[i]);
        }
      } else {
        // encoder part: A = 2^(t - L_m), dS = A (<dZ_m, V_n> - gamma_m), dV += A dZ_m
        const float a = ex2_mufu(s - sLm[j]);
        float ds = a * (row_sum<TPR>(dot16(vv, aj)) - sG[j]);
#pragma unroll
        for (int i = 0; i < kDH; ++i) accB[i] = fmaf(a, aj[i], accB[i]);
        if (MODE == kTokFull) {
          // decoder part: P = 2^(t - L_n), dS += P (<dY_n, Z_m> - delta_n)
          float zj[kDH];
          lds16(zj, sZ + j * D + part * kDH);
          const float pw = ex2_mufu(s - ln);
          ds = fmaf(pw, row_sum<TPR>(dot16(dyv, zj)) - dl, ds);
        }
#pragma unroll
        for (int i = 0; i < kDH; ++i) accA[i] = fmaf(ds, qj[i], accA[i]);
      }
    }
  }

  if (MODE == kTokStats) {
    // every thread (also past N) reaches the shuffle; l >= 1 here
    const float inv = 1.f / l;
    float y[kDH];
#pragma unroll
    for (int i = 0; i < kDH; ++i) y[i] = accA[i] * inv;
    const float delta = row_sum<TPR>(dot16(dyv, y));
    if (in_range && part == 0) {
      p.ltok[tok] = valid ? mx + __log2f(l) : 0.f;
      p.dtok[tok] = valid ? delta : 0.f;
    }
    return;
  }
  if (!in_range) return;
  // dK = scale sum dS q = ln2 sum dS (scale log2(e) q); masked tokens get zeros
#pragma unroll
  for (int i = 0; i < kDH; ++i) {
    accA[i] = valid ? accA[i] * kLn2 : 0.f;
    accB[i] = valid ? accB[i] : 0.f;
  }
  if (p.g32 != nullptr) {
    float* o = p.g32 + (static_cast<size_t>(b) * p.N + n) * p.g_ld + h * D + part * kDH;
    float4* ok = reinterpret_cast<float4*>(o + p.g_col_k);
    float4* ov = reinterpret_cast<float4*>(o + p.g_col_v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      ok[i] = make_float4(accA[4 * i], accA[4 * i + 1], accA[4 * i + 2], accA[4 * i + 3]);
      ov[i] = make_float4(accB[4 * i], accB[4 * i + 1], accB[4 * i + 2], accB[4 * i + 3]);
    }
  } else {
    uint4* ok = reinterpret_cast<uint4*>(p.dk16 + tok * D + part * kDH);
    uint4* ov = reinterpret_cast<uint4*>(p.dv16 + tok * D + part * kDH);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      ok[i] = make_uint4(pack_bf16x2(accA[8 * i], accA[8 * i + 1]), pack_bf16x2(accA[8 * i + 2], accA[8 * i + 3]),
                         pack_bf16x2(accA[8 * i + 4], accA[8 * i + 5]), pack_bf16x2(accA[8 * i + 6], accA[8 * i + 7]));
      ov[i] = make_uint4(pack_bf16x2(accB[8 * i], accB[8 * i + 1]), pack_bf16x2(accB[8 * i + 2], accB[8 * i + 3]),
                         pack_bf16x2(accB[8 * i + 4], accB[8 * i + 5]), pack_bf16x2(accB[8 * i + 6], accB[8 * i + 7]));
    }
  }
}

// ---------------------------------------------------------------------------
// Projection gradients (eq. 7 and 9 run backwards): 64 x 64 output tiles,
// 16-deep shared-memory k-steps, 4 x 4 outputs per thread.
// ---------------------------------------------------------------------------
constexpr int kTK = 16;
constexpr int kPad = 4;

// dX[r][c] = sum_j G[r][j] Wcat[c][j], Wcat = [W_0 | W_1 | ...] (each [C][C]).
__global__ void __launch_bounds__(256) dx_kernel(const DxParams p) {
  constexpr int TM = kBwdGemmTile, TN = kBwdGemmTile;
  __shared__ float sG[kTK][TM + kPad];
  __shared__ float sW[kTK][TN + kPad];
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  const long r0 = static_cast<long>(blockIdx.x) * TM;
  const int c0 = blockIdx.y * TN;
  const int J = p.nw * p.C;
  float acc[4][4] = {};
  for (int j0 = 0; j0 < J; j0 += kTK) {
    const int q = j0 / p.C, jj0 = j0 % p.C;
    for (int e = threadIdx.x; e < TM * kTK; e += blockDim.x) {
      const int r = e / kTK, k = e % kTK;
      const long gr = r0 + r;
      sG[k][r] = gr < p.R ? p.g[gr * J + j0 + k] : 0.f;
    }
    for (int e = threadIdx.x; e < TN * kTK; e += blockDim.x) {
      const int c = e / kTK, k = e % kTK;
      sW[k][c] = c0 + c < p.C ? bf(p.w[q][static_cast<size_t>(c0 + c) * p.C + jj0 + k]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < kTK; ++k) {
      float a[4], w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = sG[k][ty + 16 * i];
        w[i] = sW[k][tx + 16 * i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], w[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const long r = r0 + ty + 16 * i;
    if (r >= p.R) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = c0 + tx + 16 * j;
      if (c < p.C) p.dx[r * p.C + c] = to_bf16(acc[i][j]);
    }
  }
}

// part[split][c][j] = sum over the split's rows r of X[r][c] G[r][j].
__global__ void __launch_bounds__(256) dw_kernel(const DwParams p) {
  constexpr int TM = kBwdGemmTile, TN = kBwdGemmTile;
  __shared__ float sX[kTK][TM + kPad];
  __shared__ float sG[kTK][TN + kPad];
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  const int c0 = blockIdx.x * TM, j0 = blockIdx.y * TN, split = blockIdx.z;
  const long rs = static_cast<long>(split) * kBwdDwRows;
  const long re = min(rs + kBwdDwRows, static_cast<long>(p.R));
  float acc[4][4] = {};
  for (long r = rs; r < re; r += kTK) {
    for (int e = threadIdx.x; e < kTK * TM; e += blockDim.x) {
      const int k = e / TM, c = e % TM;
      const long rr = r + k;
      sX[k][c] = (rr < re && c0 + c < p.C) ? bf(p.x[rr * p.C + c0 + c]) : 0.f;
    }
    for (int e = threadIdx.x; e < kTK * TN; e += blockDim.x) {
      const int k = e / TN, j = e % TN;
      const long rr = r + k;
      sG[k][j] = (rr < re && j0 + j < p.J) ? p.g[rr * p.J + j0 + j] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < kTK; ++k) {
      float a[4], w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = sX[k][ty + 16 * i];
        w[i] = sG[k][tx + 16 * i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], w[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int c = c0 + ty + 16 * i;
    if (c >= p.C) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int jj = j0 + tx + 16 * j;
      if (jj < p.J) p.part[(static_cast<size_t>(split) * p.C + c) * p.J + jj] = acc[i][j];
    }
  }
}

__global__ void __launch_bounds__(256) dw_reduce_kernel(const DwReduceParams p) {
  const int ncols = p.shared ? 2 * p.C : p.J;
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= p.C * ncols) return;
  const int c = idx / ncols, j = idx % ncols;
  float s = 0.f;
  for (int sp = 0; sp < p.n_splits; ++sp) {
    const float* row = p.part + (static_cast<size_t>(sp) * p.C + c) * p.J;
    s += row[j];
    if (p.shared) s += row[j + 2 * p.C];
  }
  const int q = j / p.C, jj = j % p.C;
  if (p.dw[q]) p.dw[q][static_cast<size_t>(c) * p.C + jj] = s;
  if (p.shared && p.dw[q + 2]) p.dw[q + 2][static_cast<size_t>(c) * p.C + jj] = s;
}

__global__ void __launch_bounds__(256) cvt_kernel(const CvtParams p) {
  const long i = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < p.n) p.dst[i] = bf(p.src[i]);
}

unsigned blocks_for(long n, int threads) { return static_cast<unsigned>((n + threads - 1) / threads); }

}  // namespace

cudaError_t launch_lat(int mode, const LatParams& p, cudaStream_t s) {
  const dim3 grid(p.n_splits, (p.M + p.rows_per_block - 1) / p.rows_per_block, p.B * p.H);
  const int threads = p.rows_per_block * (p.D / kDH);
#define FLARE_LAT(DD, MM) lat_kernel<DD, MM><<<grid, threads, 0, s>>>(p)
  if (p.D == 16) {
    if (mode == kLatForward) FLARE_LAT(16, kLatForward);
    else if (mode == kLatDecoder) FLARE_LAT(16, kLatDecoder);
    else FLARE_LAT(16, kLatEncoder);
  } else {
    if (mode == kLatForward) FLARE_LAT(32, kLatForward);
    else if (mode == kLatDecoder) FLARE_LAT(32, kLatDecoder);
    else FLARE_LAT(32, kLatEncoder);
  }
#undef FLARE_LAT
  return cudaGetLastError();
}

cudaError_t launch_lat_merge(const LatMergeParams& p, cudaStream_t s) {
  const unsigned grid = blocks_for(static_cast<long>(p.BH) * p.M, 256);
  if (p.D == 16) lat_merge_kernel<16><<<grid, 256, 0, s>>>(p);
  else lat_merge_kernel<32><<<grid, 256, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_lat_sum(const LatSumParams& p, cudaStream_t s) {
  const long rows = static_cast<long>(p.fold_batch ? p.H : p.B * p.H) * p.M;
  const unsigned grid = blocks_for(rows, 128);
  if (p.D == 16) lat_sum_kernel<16><<<grid, 128, 0, s>>>(p);
  else lat_sum_kernel<32><<<grid, 128, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_tok(int mode, const TokParams& p, cudaStream_t s) {
  const dim3 grid((p.N + kBwdTokBlock - 1) / kBwdTokBlock, p.B * p.H);
  const int threads = kBwdTokBlock * (p.D / kDH);
#define FLARE_TOK(DD, MM) tok_kernel<DD, MM><<<grid, threads, 0, s>>>(p)
  if (p.D == 16) {
    if (mode == kTokStats) FLARE_TOK(16, kTokStats);
    else if (mode == kTokFull) FLARE_TOK(16, kTokFull);
    else FLARE_TOK(16, kTokEncoder);
  } else {
    if (mode == kTokStats) FLARE_TOK(32, kTokStats);
    else if (mode == kTokFull) FLARE_TOK(32, kTokFull);
    else FLARE_TOK(32, kTokEncoder);
  }
#undef FLARE_TOK
  return cudaGetLastError();
}

cudaError_t launch_dx(const DxParams& p, cudaStream_t s) {
  const dim3 grid(blocks_for(p.R, kBwdGemmTile), blocks_for(p.C, kBwdGemmTile));
  dx_kernel<<<grid, 256, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_dw(const DwParams& p, cudaStream_t s) {
  const dim3 grid(blocks_for(p.C, kBwdGemmTile), blocks_for(p.J, kBwdGemmTile), p.n_splits);
  dw_kernel<<<grid, 256, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_dw_reduce(const DwReduceParams& p, cudaStream_t s) {
  const long n = static_cast<long>(p.C) * (p.shared ? 2 * p.C : p.J);
  dw_reduce_kernel<<<blocks_for(n, 256), 256, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_cvt(const CvtParams& p, cudaStream_t s) {
  cvt_kernel<<<blocks_for(p.n, 256), 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace flare
