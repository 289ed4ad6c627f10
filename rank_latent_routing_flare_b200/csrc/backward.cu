// Gradient kernels of the FLARE / FLARE++ mixer: the score and gradient
// products on the tensor cores (mma.sync, tf32 operands, fp32 accumulation),
// softmax weights, normalisers and every reduction in fp32.
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
// Kernels (template arguments <D, mode, 16-row tiles per warp>):
//   lat_kernel<., kLatForward, 1>    encoder recompute partials (max, sum, sum w v)
//   lat_merge_kernel                 Z and the encoder row log-normalisers
//   tok_kernel<., kTokStats, 1>      decoder per-token log-normaliser and delta
//   lat_kernel<., kLatDecoder, .>    dZ = P^T dY and the decoder's dQ (per split)
//   lat_sum_kernel                   fixed-order sums of split partials (+ gamma)
//   pad_kernel                       padded tf32 images of Q, Z, dZ for the token pass
//   tok_kernel<., kTokFull, .>       dK (decoder + encoder) and dV
//   lat_kernel<., kLatEncoder, .>    the encoder's dQ (per split)
//   tok_kernel<., kTokEncoder, .>    dK, dV of the query synthesis
// Every reduction has a fixed order: the results are bitwise reproducible.
// No kernel waits on another CTA or on a flag: there are no spin loops.
#include "bwd_internal.h"
#include "flare_internal.h"
#include "ptx.cuh"

namespace flare {
namespace {

constexpr unsigned kAll = 0xffffffffu;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ float bf(uint16_t x) { return __uint_as_float(static_cast<uint32_t>(x) << 16); }

// ---------------------------------------------------------------------------
// Tensor-core fragments: mma.sync m16n8k8 with tf32 operands and fp32
// accumulation.  lane = 4 g + t.  A (16 x 8): a0 (g, t), a1 (g+8, t),
// a2 (g, t+4), a3 (g+8, t+4).  B (8 x 8): b0 (k t, n g), b1 (k t+4, n g).
// C (16 x 8): c0 (g, 2t), c1 (g, 2t+1), c2 (g+8, 2t), c3 (g+8, 2t+1).
// A C tile is reused as the A operand of a second product (over its 8
// columns) with the k order permuted: A'[.][t] = C[.][2t] and
// A'[.][t+4] = C[.][2t+1]; the B operand then takes rows 2t and 2t+1.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}

__device__ __forceinline__ void mma8(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// A operand from a C tile (k order permuted as above), rounded to tf32.
__device__ __forceinline__ void c_as_a(uint32_t (&a)[4], float c0, float c1, float c2, float c3) {
  a[0] = tf32(c0);
  a[1] = tf32(c2);
  a[2] = tf32(c1);
  a[3] = tf32(c3);
}

__device__ __forceinline__ uint32_t fbits(const float* p) { return __float_as_uint(*p); }

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem)), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// Quad (the 4 lanes of one fragment row) reductions.
__device__ __forceinline__ float quad_max(float x) {
  x = fmaxf(x, __shfl_xor_sync(kAll, x, 1));
  return fmaxf(x, __shfl_xor_sync(kAll, x, 2));
}
__device__ __forceinline__ float quad_sum(float x) {
  x += __shfl_xor_sync(kAll, x, 1);
  return x + __shfl_xor_sync(kAll, x, 2);
}

// Stages rows [0, rows) of a [rows][D] operand into shared memory (row
// stride LD floats), tf32-rounded, scaled by `mul`; rows >= valid are zero.
template <int D, int LD>
__device__ __forceinline__ void stage_f32(float* dst, const float* src, int rows, int valid, float mul) {
  for (int i = threadIdx.x; i < rows * D; i += blockDim.x) {
    const int r = i / D, c = i - r * D;
    dst[r * LD + c] = r < valid ? __uint_as_float(tf32(mul * src[i])) : 0.f;
  }
}
template <int D, int LD>
__device__ __forceinline__ void stage_bf16(float* dst, const uint16_t* src, int rows, int valid) {
  for (int i = threadIdx.x; i < rows * D; i += blockDim.x) {
    const int r = i / D, c = i - r * D;
    dst[r * LD + c] = r < valid ? bf(src[i]) : 0.f;  // bf16 values are exact in tf32
  }
}

// ---------------------------------------------------------------------------
// Latent-parallel pass: a warp owns MT tiles of 16 latent rows of one head and
// one token split (MT = 2 shares every B fragment between two MMAs; the
// forward mode keeps MT = 1 for its online softmax), and walks the split's
// valid tokens in tiles of 64 that the CTA stages in shared memory (double
// buffered).  Per tile and 8-token column block:
// scores S = smul (qmul Q) K^T on the tensor cores (qmul smul = scale log2(e);
// the forward mode takes smul = 1), then
//   forward:  online softmax over tokens, O += 2^(S - max) V
//   decoder:  W = 2^(S - L_n), dS = W (Z dY^T - delta_n), dZ += W dY, dQ += dS K
//   encoder:  W = 2^(S - L_m), dS = W (dZ V^T - gamma_m), dQ += dS K
// ---------------------------------------------------------------------------
template <int D, int MODE, int MT>
__global__ void __launch_bounds__(256) lat_kernel(const LatParams p) {
  static_assert(MODE != kLatForward || MT == 1, "the online softmax keeps one m-tile per warp");
  constexpr int KS = D / 8, LD = D + 4, T = kBwdTokTile, NT = T / 8;
  // two buffers: the next tile is loaded into registers while this one is
  // used, and stored after it (one barrier per tile)
  constexpr int PV = (T * D / 8 + 63) / 64;  // 16-byte words per thread and operand (>= 64 threads)
  __shared__ __align__(16) float sKb[2][T * LD];
  __shared__ __align__(16) float sXb[2][T * LD];  // V (forward, encoder) or dY (decoder)
  __shared__ float sLb[2][T], sDlb[2][T];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int split = blockIdx.x, bh = blockIdx.z;
  const int b = bh / p.H, h = bh % p.H;
  const int gq = p.q_per_batch ? bh : h;
  bool bad = false;
  const int L = shard_valid_len(p.lengths, b, p.N, p.tok_offset, p.n_global, &bad);
  if (bad && threadIdx.x == 0 && split == 0 && blockIdx.y == 0) atomicOr(p.err, FLARE_DEV_BAD_LENGTH);
  const int ntv = (L + T - 1) / T;
  const int t_begin = split * p.tiles_per_split;
  const int t_end = min(t_begin + p.tiles_per_split, ntv);

  // this thread's latent rows: m-tile mt of the warp, rows g (i = 0), g + 8 (i = 1)
  int mr[MT][2];
  bool act[MT][2];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      mr[mt][i] = blockIdx.y * p.rows_per_block + (warp * MT + mt) * 16 + g + 8 * i;
      act[mt][i] = mr[mt][i] < p.M;
    }
  // A fragments: log2-scaled queries, and Z (decoder) or dZ (encoder); rows
  // past M are zero and write nothing
  uint32_t qa[MT][KS][4], za[MT][KS][4];
  float lr[MT][2], gr[MT][2];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
    const float* qrow[2];
    const float* zrow[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int m = act[mt][i] ? mr[mt][i] : 0;
      qrow[i] = p.q + (static_cast<size_t>(gq) * p.M + m) * D;
      zrow[i] = p.zrow + (static_cast<size_t>(bh) * p.M + m) * D;
      lr[mt][i] = (MODE == kLatEncoder && act[mt][i]) ? p.lrow[static_cast<size_t>(bh) * p.M + m] : 0.f;
      gr[mt][i] = (MODE == kLatEncoder && act[mt][i]) ? p.grow[static_cast<size_t>(bh) * p.M + m] : 0.f;
    }
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      const int c = ks * 8 + t;
      qa[mt][ks][0] = act[mt][0] ? tf32(p.qmul * qrow[0][c]) : 0u;
      qa[mt][ks][1] = act[mt][1] ? tf32(p.qmul * qrow[1][c]) : 0u;
      qa[mt][ks][2] = act[mt][0] ? tf32(p.qmul * qrow[0][c + 4]) : 0u;
      qa[mt][ks][3] = act[mt][1] ? tf32(p.qmul * qrow[1][c + 4]) : 0u;
      if (MODE != kLatForward) {
        za[mt][ks][0] = act[mt][0] ? tf32(zrow[0][c]) : 0u;
        za[mt][ks][1] = act[mt][1] ? tf32(zrow[1][c]) : 0u;
        za[mt][ks][2] = act[mt][0] ? tf32(zrow[0][c + 4]) : 0u;
        za[mt][ks][3] = act[mt][1] ? tf32(zrow[1][c + 4]) : 0u;
      }
    }
  }
  float oa[MT][KS][4], ob[MT][KS][4];  // forward: O; decoder: dZ (oa), dQ (ob); encoder: dQ (ob)
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int nd = 0; nd < KS; ++nd)
#pragma unroll
      for (int i = 0; i < 4; ++i) oa[mt][nd][i] = ob[mt][nd][i] = 0.f;
  float mx0 = -INFINITY, mx1 = -INFINITY, l0 = 0.f, l1 = 0.f;  // forward (MT == 1)

  const uint16_t* kh = p.k + static_cast<size_t>(bh) * p.N * D;
  const uint16_t* xh = (MODE == kLatDecoder ? p.dy : p.v) + static_cast<size_t>(bh) * p.N * D;
  uint4 pk[PV], px[PV];
  float pl = 0.f, pd = 0.f;
  auto fetch = [&](int tile) {  // global -> registers; tokens past L are zero
    const int n0 = tile * T, nv = min(T, L - n0);
    const uint4* k16 = reinterpret_cast<const uint4*>(kh + static_cast<size_t>(n0) * D);
    const uint4* x16 = reinterpret_cast<const uint4*>(xh + static_cast<size_t>(n0) * D);
#pragma unroll
    for (int u = 0; u < PV; ++u) {
      const int i = threadIdx.x + u * blockDim.x;
      const bool in = i < T * D / 8 && (i * 8) / D < nv;
      pk[u] = in ? k16[i] : make_uint4(0u, 0u, 0u, 0u);
      px[u] = in ? x16[i] : make_uint4(0u, 0u, 0u, 0u);
    }
    if (MODE == kLatDecoder && threadIdx.x < T) {
      const size_t o = static_cast<size_t>(bh) * p.N + n0 + threadIdx.x;
      pl = static_cast<int>(threadIdx.x) < nv ? p.ltok[o] : 0.f;
      pd = static_cast<int>(threadIdx.x) < nv ? p.dtok[o] : 0.f;
    }
  };
  auto commit = [&](int buf) {  // registers -> shared memory (fp32; bf16 values are exact in tf32)
#pragma unroll
    for (int u = 0; u < PV; ++u) {
      const int i = threadIdx.x + u * blockDim.x;
      if (i >= T * D / 8) continue;
      const int e = i * 8, r = e / D, c = e - r * D;
      const uint32_t wk[4] = {pk[u].x, pk[u].y, pk[u].z, pk[u].w};
      const uint32_t wx[4] = {px[u].x, px[u].y, px[u].z, px[u].w};
      float4* dk = reinterpret_cast<float4*>(&sKb[buf][r * LD + c]);
      float4* dx = reinterpret_cast<float4*>(&sXb[buf][r * LD + c]);
      dk[0] = make_float4(bf16_lo(wk[0]), bf16_hi(wk[0]), bf16_lo(wk[1]), bf16_hi(wk[1]));
      dk[1] = make_float4(bf16_lo(wk[2]), bf16_hi(wk[2]), bf16_lo(wk[3]), bf16_hi(wk[3]));
      dx[0] = make_float4(bf16_lo(wx[0]), bf16_hi(wx[0]), bf16_lo(wx[1]), bf16_hi(wx[1]));
      dx[1] = make_float4(bf16_lo(wx[2]), bf16_hi(wx[2]), bf16_lo(wx[3]), bf16_hi(wx[3]));
    }
    if (MODE == kLatDecoder && threadIdx.x < T) {
      sLb[buf][threadIdx.x] = pl;
      sDlb[buf][threadIdx.x] = pd;
    }
  };
  if (t_begin < t_end) {
    fetch(t_begin);
    commit(0);
  }
  __syncthreads();
  for (int tile = t_begin; tile < t_end; ++tile) {
    const int buf = (tile - t_begin) & 1;
    const int n0 = tile * T;
    const int nv = min(T, L - n0);
    const bool more = tile + 1 < t_end;
    if (more) fetch(tile + 1);
    const float* sK = sKb[buf];
    const float* sX = sXb[buf];
    const float* sL = sLb[buf];
    const float* sDl = sDlb[buf];

    if (MODE == kLatForward) {
      float s[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int i = 0; i < 4; ++i) s[nt][i] = 0.f;
        const float* kr = sK + (nt * 8 + g) * LD;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) mma8(s[nt], qa[0][ks], fbits(kr + ks * 8 + t), fbits(kr + ks * 8 + t + 4));
      }
      float tm0 = -INFINITY, tm1 = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int ca = nt * 8 + 2 * t;
        if (ca >= nv) { s[nt][0] = -INFINITY; s[nt][2] = -INFINITY; }
        if (ca + 1 >= nv) { s[nt][1] = -INFINITY; s[nt][3] = -INFINITY; }
        tm0 = fmaxf(tm0, fmaxf(s[nt][0], s[nt][1]));
        tm1 = fmaxf(tm1, fmaxf(s[nt][2], s[nt][3]));
      }
      tm0 = quad_max(tm0);
      tm1 = quad_max(tm1);
      const float nm0 = fmaxf(mx0, tm0), nm1 = fmaxf(mx1, tm1);  // finite: the tile holds a valid token
      const float r0 = ex2_mufu(mx0 - nm0), r1 = ex2_mufu(mx1 - nm1);
      mx0 = nm0;
      mx1 = nm1;
      l0 *= r0;
      l1 *= r1;
#pragma unroll
      for (int nd = 0; nd < KS; ++nd) {
        oa[0][nd][0] *= r0; oa[0][nd][1] *= r0;
        oa[0][nd][2] *= r1; oa[0][nd][3] *= r1;
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const float p0 = ex2_mufu(s[nt][0] - nm0), p1 = ex2_mufu(s[nt][1] - nm0);
        const float p2 = ex2_mufu(s[nt][2] - nm1), p3 = ex2_mufu(s[nt][3] - nm1);
        l0 += p0 + p1;
        l1 += p2 + p3;
        uint32_t pa[4];
        c_as_a(pa, p0, p1, p2, p3);
        const float* v0 = sX + (nt * 8 + 2 * t) * LD + g;
#pragma unroll
        for (int nd = 0; nd < KS; ++nd) mma8(oa[0][nd], pa, fbits(v0 + nd * 8), fbits(v0 + LD + nd * 8));
      }
    } else {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        // B fragments of this 8-token block, shared by the warp's m-tiles
        uint32_t bs[KS][2], bg[KS][2], bk[KS][2], by[KS][2];
        const float* kr = sK + (nt * 8 + g) * LD;
        const float* xr = sX + (nt * 8 + g) * LD;
        const float* k0 = sK + (nt * 8 + 2 * t) * LD + g;
        const float* y0 = sX + (nt * 8 + 2 * t) * LD + g;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          bs[ks][0] = fbits(kr + ks * 8 + t);
          bs[ks][1] = fbits(kr + ks * 8 + t + 4);
          bg[ks][0] = fbits(xr + ks * 8 + t);
          bg[ks][1] = fbits(xr + ks * 8 + t + 4);
          bk[ks][0] = fbits(k0 + ks * 8);
          bk[ks][1] = fbits(k0 + LD + ks * 8);
          if (MODE == kLatDecoder) {
            by[ks][0] = fbits(y0 + ks * 8);
            by[ks][1] = fbits(y0 + LD + ks * 8);
          }
        }
        const int ca = nt * 8 + 2 * t;
        const bool va = ca < nv, vb = ca + 1 < nv;
        float la = 0.f, lb = 0.f, da = 0.f, db = 0.f;
        if (MODE == kLatDecoder) {
          la = sL[ca];
          lb = sL[ca + 1];
          da = sDl[ca];
          db = sDl[ca + 1];
        }
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          float s[4] = {0.f, 0.f, 0.f, 0.f}, gg[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int ks = 0; ks < KS; ++ks) {
            mma8(s, qa[mt][ks], bs[ks][0], bs[ks][1]);
            mma8(gg, za[mt][ks], bg[ks][0], bg[ks][1]);
          }
          float w[4], ds[4];
          if (MODE == kLatDecoder) {
            // W = 2^(S - L_n) per token column, dS = W (<Z_m, dY_n> - delta_n)
            w[0] = va ? ex2_mufu(fmaf(s[0], p.smul, -la)) : 0.f;
            w[1] = vb ? ex2_mufu(fmaf(s[1], p.smul, -lb)) : 0.f;
            w[2] = va ? ex2_mufu(fmaf(s[2], p.smul, -la)) : 0.f;
            w[3] = vb ? ex2_mufu(fmaf(s[3], p.smul, -lb)) : 0.f;
            ds[0] = w[0] * (gg[0] - da);
            ds[1] = w[1] * (gg[1] - db);
            ds[2] = w[2] * (gg[2] - da);
            ds[3] = w[3] * (gg[3] - db);
            uint32_t wa[4];
            c_as_a(wa, w[0], w[1], w[2], w[3]);
#pragma unroll
            for (int nd = 0; nd < KS; ++nd) mma8(oa[mt][nd], wa, by[nd][0], by[nd][1]);
          } else {
            // W = 2^(S - L_m) per latent row, dS = W (<dZ_m, V_n> - gamma_m)
            w[0] = va ? ex2_mufu(fmaf(s[0], p.smul, -lr[mt][0])) : 0.f;
            w[1] = vb ? ex2_mufu(fmaf(s[1], p.smul, -lr[mt][0])) : 0.f;
            w[2] = va ? ex2_mufu(fmaf(s[2], p.smul, -lr[mt][1])) : 0.f;
            w[3] = vb ? ex2_mufu(fmaf(s[3], p.smul, -lr[mt][1])) : 0.f;
            ds[0] = w[0] * (gg[0] - gr[mt][0]);
            ds[1] = w[1] * (gg[1] - gr[mt][0]);
            ds[2] = w[2] * (gg[2] - gr[mt][1]);
            ds[3] = w[3] * (gg[3] - gr[mt][1]);
          }
          uint32_t da4[4];
          c_as_a(da4, ds[0], ds[1], ds[2], ds[3]);
#pragma unroll
          for (int nd = 0; nd < KS; ++nd) mma8(ob[mt][nd], da4, bk[nd][0], bk[nd][1]);
        }
      }
    }
    if (more) commit(buf ^ 1);
    __syncthreads();
  }

  // partials of rows mr[mt][0] (c0, c1) and mr[mt][1] (c2, c3)
  if (MODE == kLatForward) {
    l0 = quad_sum(l0);
    l1 = quad_sum(l1);
    const float mx[2] = {mx0, mx1}, ll[2] = {l0, l1};
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      if (!act[0][i]) continue;
      float* o = p.part_a + ((static_cast<size_t>(bh) * p.n_splits + split) * p.M + mr[0][i]) * (D + 2);
      if (t == 0) {
        o[0] = mx[i];
        o[1] = ll[i];
      }
#pragma unroll
      for (int nd = 0; nd < KS; ++nd) {
        const int c = 2 + nd * 8 + 2 * t;
        o[c] = oa[0][nd][2 * i];
        o[c + 1] = oa[0][nd][2 * i + 1];
      }
    }
  } else {
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        if (!act[mt][i]) continue;
        const size_t base = (static_cast<size_t>(bh) * p.n_splits + split) * p.M + mr[mt][i];
#pragma unroll
        for (int nd = 0; nd < KS; ++nd) {
          const int c = nd * 8 + 2 * t;
          if (MODE == kLatDecoder)
            *reinterpret_cast<float2*>(p.part_a + base * D + c) = make_float2(oa[mt][nd][2 * i], oa[mt][nd][2 * i + 1]);
          *reinterpret_cast<float2*>(p.part_b + base * D + c) = make_float2(ob[mt][nd][2 * i], ob[mt][nd][2 * i + 1]);
        }
      }
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
  // splits in ascending (rank, split) order
  float G = -INFINITY;
  for (int j = 0; j < p.R * p.S; ++j) {
    const float* e = base + (j / p.S) * p.rank_stride + (j % p.S) * sstride;
    if (e[1] > 0.f) G = fmaxf(G, e[0]);
  }
  float den = 0.f, acc[D];
#pragma unroll
  for (int d = 0; d < D; ++d) acc[d] = 0.f;
  for (int j = 0; j < p.R * p.S; ++j) {
    const float* e = base + (j / p.S) * p.rank_stride + (j % p.S) * sstride;
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
      for (int j = 0; j < p.R * p.S; ++j) {  // ascending (rank, split)
        const int s = j % p.S;
        const float4* e = reinterpret_cast<const float4*>(part + (j / p.S) * p.rank_stride +
                                                          ((static_cast<size_t>(bh) * p.S + s) * p.M + m) * D);
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
    if (p.addend) acc[d] += p.addend[static_cast<size_t>(r) * D + d];
    p.out[static_cast<size_t>(r) * D + d] = acc[d];
    if (p.zref) gsum = fmaf(acc[d], p.zref[static_cast<size_t>(r) * D + d], gsum);
  }
  if (p.zref) p.gamma[r] = gsum;
}

// ---------------------------------------------------------------------------
// Token-parallel pass: a warp owns MT tiles of 16 token rows (a CTA 128 tokens)
// of one head and walks all latents in chunks of 64 (32 for D = 32), copied
// with cp.async from padded tf32 images into two shared-memory buffers.
// Per 8-latent column block, on the tensor cores: S = smul K (qpad's Q)^T, and
//   stats:    online softmax over latents, Y += 2^(S - max) Z; at the end
//             L_n = log2 sum 2^S and delta_n = <dY_n, Y_n>
//   full:     A = 2^(S - L_m), P = 2^(S - L_n), dA = V dZ^T, dP = dY Z^T,
//             dS = A (dA - gamma_m) + P (dP - delta_n), dK += dS (c Q),
//             dV += A dZ
//   encoder:  the A terms alone (query synthesis: no decoder)
// ---------------------------------------------------------------------------
template <int D, int MODE, int MT>
__global__ void __launch_bounds__(256) tok_kernel(const TokParams p) {
  constexpr int KS = D / 8, LD = D + 4, MC = tok_chunk(D);
  // two chunk buffers, filled by cp.async from the padded tf32 copies while
  // the other chunk is used (one barrier per chunk)
  __shared__ __align__(16) float sQb[2][MC * LD];  // log2-scaled queries
  __shared__ __align__(16) float sAb[2][MC * LD];  // Z (stats) or dZ
  __shared__ __align__(16) float sZb[2][MC * LD];  // Z (full)
  __shared__ __align__(16) float sLmb[2][MC], sGb[2][MC];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int bh = blockIdx.y, b = bh / p.H, h = bh % p.H;
  const int gq = p.q_per_batch ? bh : h;
  bool bad = false;
  const int L = shard_valid_len(p.lengths, b, p.N, p.tok_offset, p.n_global, &bad);
  // this thread's token rows: m-tile mt of the warp, rows g (i = 0) and g + 8 (i = 1)
  int rr[MT][2];
  bool in[MT][2];
  size_t tk[MT][2];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      rr[mt][i] = blockIdx.x * kBwdTokBlock + (warp * MT + mt) * 16 + g + 8 * i;
      in[mt][i] = rr[mt][i] < p.N;
      tk[mt][i] = static_cast<size_t>(bh) * p.N + (in[mt][i] ? rr[mt][i] : 0);
    }

  const float* qpad = p.qpad + static_cast<size_t>(gq) * p.M * LD;
  const float* apad = (MODE == kTokStats ? p.zpad : p.dzpad) + static_cast<size_t>(bh) * p.M * LD;
  const float* zpad = p.zpad + static_cast<size_t>(bh) * p.M * LD;
  const float* lmh = p.lm + static_cast<size_t>(bh) * p.M;
  const float* gmh = p.gam + static_cast<size_t>(bh) * p.M;
  auto issue = [&](int mb, int buf) {
    const int n16 = min(MC, p.M - mb) * LD / 4;
    for (int i = threadIdx.x; i < n16; i += blockDim.x) {
      cp_async16(&sQb[buf][4 * i], qpad + static_cast<size_t>(mb) * LD + 4 * i);
      cp_async16(&sAb[buf][4 * i], apad + static_cast<size_t>(mb) * LD + 4 * i);
      if (MODE == kTokFull) cp_async16(&sZb[buf][4 * i], zpad + static_cast<size_t>(mb) * LD + 4 * i);
    }
    if (MODE != kTokStats) {
      for (int i = threadIdx.x; i < min(MC, p.M - mb) / 4; i += blockDim.x) {
        cp_async16(&sLmb[buf][4 * i], lmh + mb + 4 * i);
        cp_async16(&sGb[buf][4 * i], gmh + mb + 4 * i);
      }
    }
    cp_async_commit();
  };
  issue(0, 0);

  // A fragments of this warp's token rows (bf16 values are exact in tf32)
  uint32_t ka[MT][KS][4], va[MT][KS][4], ya[MT][KS][4];
  auto frag = [&](const uint16_t* src, uint32_t (&f)[MT][KS][4]) {
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        const int c = ks * 8 + t;
        f[mt][ks][0] = in[mt][0] ? static_cast<uint32_t>(src[tk[mt][0] * D + c]) << 16 : 0u;
        f[mt][ks][1] = in[mt][1] ? static_cast<uint32_t>(src[tk[mt][1] * D + c]) << 16 : 0u;
        f[mt][ks][2] = in[mt][0] ? static_cast<uint32_t>(src[tk[mt][0] * D + c + 4]) << 16 : 0u;
        f[mt][ks][3] = in[mt][1] ? static_cast<uint32_t>(src[tk[mt][1] * D + c + 4]) << 16 : 0u;
      }
  };
  frag(p.k, ka);
  if (MODE != kTokStats) frag(p.v, va);
  if (MODE == kTokFull) frag(p.dy, ya);
  float ln[MT][2], dl[MT][2];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      ln[mt][i] = (MODE == kTokFull && in[mt][i]) ? p.ltok[tk[mt][i]] : 0.f;
      dl[mt][i] = (MODE == kTokFull && in[mt][i]) ? p.dtok[tk[mt][i]] : 0.f;
    }
  float oa[MT][KS][4], ob[MT][KS][4];  // stats: Y (oa); full, encoder: dK (oa), dV (ob)
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int nd = 0; nd < KS; ++nd)
#pragma unroll
      for (int i = 0; i < 4; ++i) oa[mt][nd][i] = ob[mt][nd][i] = 0.f;
  float mx0 = -INFINITY, mx1 = -INFINITY, l0 = 0.f, l1 = 0.f;  // stats (MT == 1)

  for (int mb = 0, it = 0; mb < p.M; mb += MC, ++it) {
    const int buf = it & 1;
    const int mc = min(MC, p.M - mb);  // a multiple of 16
    cp_async_wait_all();
    __syncthreads();  // chunk `it` has landed; chunk it-1 has been consumed
    if (mb + MC < p.M) issue(mb + MC, buf ^ 1);
    const float* sQ = sQb[buf];
    const float* sA = sAb[buf];
    const float* sZ = sZb[buf];
    const float* sLm = sLmb[buf];
    const float* sG = sGb[buf];
    const int ntl = mc / 8;

    if (MODE == kTokStats) {
      static_assert(MODE != kTokStats || MT == 1, "the statistics pass keeps one m-tile per warp");
      float s[MC / 8][4];
      float tm0 = -INFINITY, tm1 = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < MC / 8; ++nt) {
#pragma unroll
        for (int i = 0; i < 4; ++i) s[nt][i] = -INFINITY;
        if (nt < ntl) {
#pragma unroll
          for (int i = 0; i < 4; ++i) s[nt][i] = 0.f;
          const float* qr = sQ + (nt * 8 + g) * LD;
#pragma unroll
          for (int ks = 0; ks < KS; ++ks) mma8(s[nt], ka[0][ks], fbits(qr + ks * 8 + t), fbits(qr + ks * 8 + t + 4));
        }
        tm0 = fmaxf(tm0, fmaxf(s[nt][0], s[nt][1]));
        tm1 = fmaxf(tm1, fmaxf(s[nt][2], s[nt][3]));
      }
      tm0 = quad_max(tm0);
      tm1 = quad_max(tm1);
      // running maximum of the unscaled products (smul > 0 keeps the order)
      const float nm0 = fmaxf(mx0, tm0), nm1 = fmaxf(mx1, tm1);
      const float q0 = ex2_mufu((mx0 - nm0) * p.smul), q1 = ex2_mufu((mx1 - nm1) * p.smul);
      const float b0 = nm0 * p.smul, b1 = nm1 * p.smul;
      mx0 = nm0;
      mx1 = nm1;
      l0 *= q0;
      l1 *= q1;
#pragma unroll
      for (int nd = 0; nd < KS; ++nd) {
        oa[0][nd][0] *= q0; oa[0][nd][1] *= q0;
        oa[0][nd][2] *= q1; oa[0][nd][3] *= q1;
      }
#pragma unroll
      for (int nt = 0; nt < MC / 8; ++nt) {
        if (nt < ntl) {
          const float p0 = ex2_mufu(fmaf(s[nt][0], p.smul, -b0)), p1 = ex2_mufu(fmaf(s[nt][1], p.smul, -b0));
          const float p2 = ex2_mufu(fmaf(s[nt][2], p.smul, -b1)), p3 = ex2_mufu(fmaf(s[nt][3], p.smul, -b1));
          l0 += p0 + p1;
          l1 += p2 + p3;
          uint32_t pa[4];
          c_as_a(pa, p0, p1, p2, p3);
          const float* z0 = sA + (nt * 8 + 2 * t) * LD + g;
#pragma unroll
          for (int nd = 0; nd < KS; ++nd) mma8(oa[0][nd], pa, fbits(z0 + nd * 8), fbits(z0 + LD + nd * 8));
        }
      }
    } else {
#pragma unroll
      for (int nt = 0; nt < MC / 8; ++nt) {
        if (nt >= ntl) continue;
        // B fragments of this 8-latent block, shared by the warp's m-tiles
        uint32_t bq[KS][2], bz[KS][2], bzz[KS][2], bk[KS][2], bv[KS][2];
        const float* qr = sQ + (nt * 8 + g) * LD;
        const float* dzr = sA + (nt * 8 + g) * LD;
        const float* zr = sZ + (nt * 8 + g) * LD;
        const float* q0 = sQ + (nt * 8 + 2 * t) * LD + g;
        const float* z0 = sA + (nt * 8 + 2 * t) * LD + g;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          bq[ks][0] = fbits(qr + ks * 8 + t);
          bq[ks][1] = fbits(qr + ks * 8 + t + 4);
          bz[ks][0] = fbits(dzr + ks * 8 + t);
          bz[ks][1] = fbits(dzr + ks * 8 + t + 4);
          if (MODE == kTokFull) {
            bzz[ks][0] = fbits(zr + ks * 8 + t);
            bzz[ks][1] = fbits(zr + ks * 8 + t + 4);
          }
          bk[ks][0] = fbits(q0 + ks * 8);
          bk[ks][1] = fbits(q0 + LD + ks * 8);
          bv[ks][0] = fbits(z0 + ks * 8);
          bv[ks][1] = fbits(z0 + LD + ks * 8);
        }
        const int ca = nt * 8 + 2 * t;
        const float lma = sLm[ca], lmb = sLm[ca + 1], ga = sG[ca], gb = sG[ca + 1];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          float s[4] = {0.f, 0.f, 0.f, 0.f}, da[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int ks = 0; ks < KS; ++ks) {
            mma8(s, ka[mt][ks], bq[ks][0], bq[ks][1]);
            mma8(da, va[mt][ks], bz[ks][0], bz[ks][1]);
          }
          float a[4], ds[4];
          a[0] = ex2_mufu(fmaf(s[0], p.smul, -lma));
          a[1] = ex2_mufu(fmaf(s[1], p.smul, -lmb));
          a[2] = ex2_mufu(fmaf(s[2], p.smul, -lma));
          a[3] = ex2_mufu(fmaf(s[3], p.smul, -lmb));
          ds[0] = a[0] * (da[0] - ga);
          ds[1] = a[1] * (da[1] - gb);
          ds[2] = a[2] * (da[2] - ga);
          ds[3] = a[3] * (da[3] - gb);
          if (MODE == kTokFull) {
            float dp[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) mma8(dp, ya[mt][ks], bzz[ks][0], bzz[ks][1]);
            ds[0] = fmaf(ex2_mufu(fmaf(s[0], p.smul, -ln[mt][0])), dp[0] - dl[mt][0], ds[0]);
            ds[1] = fmaf(ex2_mufu(fmaf(s[1], p.smul, -ln[mt][0])), dp[1] - dl[mt][0], ds[1]);
            ds[2] = fmaf(ex2_mufu(fmaf(s[2], p.smul, -ln[mt][1])), dp[2] - dl[mt][1], ds[2]);
            ds[3] = fmaf(ex2_mufu(fmaf(s[3], p.smul, -ln[mt][1])), dp[3] - dl[mt][1], ds[3]);
          }
          uint32_t sa4[4], aa4[4];
          c_as_a(sa4, ds[0], ds[1], ds[2], ds[3]);
          c_as_a(aa4, a[0], a[1], a[2], a[3]);
#pragma unroll
          for (int nd = 0; nd < KS; ++nd) {
            mma8(oa[mt][nd], sa4, bk[nd][0], bk[nd][1]);
            mma8(ob[mt][nd], aa4, bv[nd][0], bv[nd][1]);
          }
        }
      }
    }
  }

  if (MODE == kTokStats) {
    // every lane reaches the shuffles; l >= 1 for every row here
    const size_t tok0 = tk[0][0], tok1 = tk[0][1];
    const bool in0 = in[0][0], in1 = in[0][1];
    l0 = quad_sum(l0);
    l1 = quad_sum(l1);
    const float i0 = 1.f / l0, i1 = 1.f / l1;
    float d0 = 0.f, d1 = 0.f;
#pragma unroll
    for (int nd = 0; nd < KS; ++nd) {
      const int c = nd * 8 + 2 * t;
      if (in0) d0 += bf(p.dy[tok0 * D + c]) * (oa[0][nd][0] * i0) + bf(p.dy[tok0 * D + c + 1]) * (oa[0][nd][1] * i0);
      if (in1) d1 += bf(p.dy[tok1 * D + c]) * (oa[0][nd][2] * i1) + bf(p.dy[tok1 * D + c + 1]) * (oa[0][nd][3] * i1);
    }
    d0 = quad_sum(d0);
    d1 = quad_sum(d1);
    if (t == 0) {
      if (in0) {
        p.ltok[tok0] = rr[0][0] < L ? mx0 * p.smul + __log2f(l0) : 0.f;
        p.dtok[tok0] = rr[0][0] < L ? d0 : 0.f;
      }
      if (in1) {
        p.ltok[tok1] = rr[0][1] < L ? mx1 * p.smul + __log2f(l1) : 0.f;
        p.dtok[tok1] = rr[0][1] < L ? d1 : 0.f;
      }
    }
    return;
  }
  // dK = scale sum dS q = ln2 smul sum dS (qpad's q); padding tokens get zeros
  const float kdk = kLn2 * p.smul;
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      if (!in[mt][i]) continue;
      const bool v = rr[mt][i] < L;
#pragma unroll
      for (int nd = 0; nd < KS; ++nd) {
        const int c = nd * 8 + 2 * t;
        const float2 kk = v ? make_float2(oa[mt][nd][2 * i] * kdk, oa[mt][nd][2 * i + 1] * kdk)
                            : make_float2(0.f, 0.f);
        const float2 vv = v ? make_float2(ob[mt][nd][2 * i], ob[mt][nd][2 * i + 1]) : make_float2(0.f, 0.f);
        if (p.ghi != nullptr) {
          const size_t o = (static_cast<size_t>(b) * p.N + rr[mt][i]) * p.g_ld + h * D + c;
          const uint32_t kh = pack_bf16x2(kk.x, kk.y), vh = pack_bf16x2(vv.x, vv.y);
          *reinterpret_cast<uint32_t*>(p.ghi + o + p.g_col_k) = kh;
          *reinterpret_cast<uint32_t*>(p.glo + o + p.g_col_k) = pack_bf16x2(kk.x - bf16_lo(kh), kk.y - bf16_hi(kh));
          *reinterpret_cast<uint32_t*>(p.ghi + o + p.g_col_v) = vh;
          *reinterpret_cast<uint32_t*>(p.glo + o + p.g_col_v) = pack_bf16x2(vv.x - bf16_lo(vh), vv.y - bf16_hi(vh));
        } else {
          *reinterpret_cast<uint32_t*>(p.dk16 + tk[mt][i] * D + c) = pack_bf16x2(kk.x, kk.y);
          *reinterpret_cast<uint32_t*>(p.dv16 + tk[mt][i] * D + c) = pack_bf16x2(vv.x, vv.y);
        }
      }
    }
}

// dst[r][0..LD) = (tf32(mul * src[r][c]) for c < D, then zeros): the padded
// shared-memory image of a chunk of rows, copied by the token-parallel pass.
__global__ void __launch_bounds__(256) pad_kernel(const PadParams p) {
  const long i = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int ld = p.D + 4;
  if (i >= p.rows * ld) return;
  const long r = i / ld;
  const int c = static_cast<int>(i - r * ld);
  p.dst[i] = c < p.D ? __uint_as_float(tf32(p.mul * p.src[r * p.D + c])) : 0.f;
}

__global__ void __launch_bounds__(256) cvt_kernel(const CvtParams p) {
  const long i = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < p.n) p.dst[i] = bf(p.src[i]);
}

// delta_n = <dY_n, Y_n>, one thread per token of a head.
template <int D>
__global__ void __launch_bounds__(256) delta_kernel(const DeltaParams p) {
  const long i = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= static_cast<long>(p.B) * p.H * p.N) return;
  const long bh = i / p.N;
  const int n = static_cast<int>(i % p.N);
  bool bad = false;
  const int L = shard_valid_len(p.lengths, static_cast<int>(bh / p.H), p.N, p.tok_offset, p.n_global, &bad);
  float d = 0.f;
  if (n < L) {
    const float4* y = reinterpret_cast<const float4*>(p.y32 + i * D);
    const uint4* g = reinterpret_cast<const uint4*>(p.dy + i * D);
#pragma unroll
    for (int u = 0; u < D / 8; ++u) {
      const uint4 gv = g[u];
      const float4 y0 = y[2 * u], y1 = y[2 * u + 1];
      d = fmaf(bf16_lo(gv.x), y0.x, d);
      d = fmaf(bf16_hi(gv.x), y0.y, d);
      d = fmaf(bf16_lo(gv.y), y0.z, d);
      d = fmaf(bf16_hi(gv.y), y0.w, d);
      d = fmaf(bf16_lo(gv.z), y1.x, d);
      d = fmaf(bf16_hi(gv.z), y1.y, d);
      d = fmaf(bf16_lo(gv.w), y1.z, d);
      d = fmaf(bf16_hi(gv.w), y1.w, d);
    }
  }
  p.dtok[i] = d;
}

// Whether a training forward left its state in the workspace.
__global__ void check_mark_kernel(const MarkParams p) {
  if (*p.mark != kTrainStateTag) atomicOr(p.err, FLARE_DEV_NO_STATE);
}

unsigned blocks_for(long n, int threads) { return static_cast<unsigned>((n + threads - 1) / threads); }

}  // namespace

cudaError_t launch_lat(int mode, const LatParams& p, cudaStream_t s) {
  if (p.rows_per_block % 32 != 0 || p.rows_per_block < 32 || p.rows_per_block > 128) return cudaErrorInvalidValue;
  // a warp per 16 latent rows (forward) or per 32 (two m-tiles sharing the B
  // fragments: the gradient modes, when the CTA keeps at least two warps)
  const dim3 grid(p.n_splits, (p.M + p.rows_per_block - 1) / p.rows_per_block, p.B * p.H);
  // two m-tiles need rows_per_block / 32 whole warps, and at least two of them
  // (the tile loads assume 64 threads); D = 32 would spill
  const bool two = mode != kLatForward && p.rows_per_block >= 64 && p.rows_per_block % 32 == 0 && p.D == 16;
  const int threads = two ? p.rows_per_block : 2 * p.rows_per_block;
#define FLARE_LAT(DD, MM, MT) lat_kernel<DD, MM, MT><<<grid, threads, 0, s>>>(p)
  if (p.D == 16) {
    if (mode == kLatForward) FLARE_LAT(16, kLatForward, 1);
    else if (mode == kLatDecoder) { if (two) FLARE_LAT(16, kLatDecoder, 2); else FLARE_LAT(16, kLatDecoder, 1); }
    else { if (two) FLARE_LAT(16, kLatEncoder, 2); else FLARE_LAT(16, kLatEncoder, 1); }
  } else {
    if (mode == kLatForward) FLARE_LAT(32, kLatForward, 1);
    else if (mode == kLatDecoder) { if (two) FLARE_LAT(32, kLatDecoder, 2); else FLARE_LAT(32, kLatDecoder, 1); }
    else { if (two) FLARE_LAT(32, kLatEncoder, 2); else FLARE_LAT(32, kLatEncoder, 1); }
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
  // a warp per 16 token rows (statistics, D = 32) or per 32 (two m-tiles
  // sharing the B fragments: the gradient modes at D = 16)
  const dim3 grid((p.N + kBwdTokBlock - 1) / kBwdTokBlock, p.B * p.H);
  const int t1 = 2 * kBwdTokBlock, t2 = kBwdTokBlock;
#define FLARE_TOK(DD, MM, MT) tok_kernel<DD, MM, MT><<<grid, (MT == 1 ? t1 : t2), 0, s>>>(p)
  if (p.D == 16) {
    if (mode == kTokStats) FLARE_TOK(16, kTokStats, 1);
    else if (mode == kTokFull) FLARE_TOK(16, kTokFull, 2);
    else FLARE_TOK(16, kTokEncoder, 2);
  } else {
    if (mode == kTokStats) FLARE_TOK(32, kTokStats, 1);
    else if (mode == kTokFull) FLARE_TOK(32, kTokFull, 1);   // two m-tiles would need ~240 registers
    else FLARE_TOK(32, kTokEncoder, 1);
  }
#undef FLARE_TOK
  return cudaGetLastError();
}

cudaError_t launch_pad(const PadParams& p, cudaStream_t s) {
  pad_kernel<<<blocks_for(p.rows * (p.D + 4), 256), 256, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_cvt(const CvtParams& p, cudaStream_t s) {
  cvt_kernel<<<blocks_for(p.n, 256), 256, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_delta(const DeltaParams& p, cudaStream_t s) {
  const unsigned grid = blocks_for(static_cast<long>(p.B) * p.H * p.N, 256);
  if (p.D == 16) delta_kernel<16><<<grid, 256, 0, s>>>(p);
  else delta_kernel<32><<<grid, 256, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_check_mark(const MarkParams& p, cudaStream_t s) {
  check_mark_kernel<<<1, 1, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace flare
