// Host entry points of the C ABI declared in include/flare.h: argument
// validation (before anything is enqueued), workspace layout, TMA tensor maps
// and the launch sequence of the FLARE / FLARE++ forward.
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "bwd_internal.h"
#include "flare.h"
#include "flare_internal.h"

namespace flare {
namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn tensor_map_encoder() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

unsigned long long wait_timeout_ns() {
  static unsigned long long t = [] {
    const char* e = std::getenv("FLARE_WAIT_TIMEOUT_NS");
    unsigned long long v = e ? std::strtoull(e, nullptr, 10) : 0ull;
    return v > 0 ? v : 4000000000ull;  // 4 s per wait
  }();
  return t;
}

// 3-D bf16 tensor map: dims (d0 innermost, d1, d2), dense, box (b0, b1, 1).
bool map3d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t b0, uint32_t b1,
           CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = tensor_map_encoder();
  if (!fn) return false;
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
  const cuuint32_t box[3] = {b0, b1, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool map2d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint32_t b0, uint32_t b1,
           CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = tensor_map_encoder();
  if (!fn) return false;
  const cuuint64_t dims[2] = {d0, d1};
  const cuuint64_t strides[1] = {d0 * 2};
  const cuuint32_t box[2] = {b0, b1};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

CUtensorMapSwizzle row_swizzle(int D) { return D == 16 ? CU_TENSOR_MAP_SWIZZLE_32B : CU_TENSOR_MAP_SWIZZLE_64B; }

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
long cdiv(long a, long b) { return (a + b - 1) / b; }

// Number of token splits of the encoder.  Cost model: the CTAs run in
// waves of `slots` (CTAs resident on the whole GPU); a wave lasts as long as
// one split (its tiles plus a fixed set-up cost worth kSplitSetupTiles
// tiles).  Depends on the sizes only, so a given problem always uses the same
// split count (and gives the same bits).
constexpr long kSplitSetupTiles = 8;
int choose_splits(long units, long ntiles, long slots) {
  const long smax = std::max(1L, std::min(ntiles, 1024L));
  int best = 1;
  long best_cost = -1;
  for (long s = 1; s <= smax; ++s) {
    const long tps = cdiv(ntiles, s);
    if (s > 1 && cdiv(ntiles, tps) < s) continue;  // same tiling as a smaller s
    const long cost = cdiv(units * s, slots) * (tps + kSplitSetupTiles);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = static_cast<int>(s);
    }
  }
  return best;
}

struct Plan {
  int S = 1, tps = 1, LB = 1;            // encoder splits, tiles per split, latent blocks
  int dec_ctas = 1, dec_tiles = 1;       // decoder CTAs per head, tiles per CTA
  int G32 = 1;
  size_t off_err = 0, off_kt = 0, off_vt = 0, off_kp = 0, off_vp = 0, off_kn_syn = 0, off_kn = 0, off_part = 0,
         off_qx32 = 0, off_qx16 = 0, off_z32 = 0, off_z16 = 0, off_fb = 0, off_ycat = 0, total = 0;
};

Plan make_plan(int variant, long B, long H, long N, long M, long D) {
  Plan p;
  const long BH = B * H;
  const long ntiles = cdiv(N, enc_tile(static_cast<int>(D)));
  p.LB = static_cast<int>(cdiv(M, kLatBlock));
  p.S = choose_splits(BH * p.LB, ntiles, static_cast<long>(kNumSM) * enc_ctas_per_sm(static_cast<int>(D)));
  p.tps = static_cast<int>(cdiv(ntiles, p.S));
  p.S = static_cast<int>(cdiv(ntiles, p.tps));
  const long dtiles = cdiv(N, kDecTile);
  long per = std::max(1L, static_cast<long>(kNumSM) * dec_ctas_per_sm(static_cast<int>(D)) / BH);
  per = std::min(per, dtiles);
  p.dec_tiles = static_cast<int>(cdiv(dtiles, per));
  p.dec_ctas = static_cast<int>(cdiv(dtiles, p.dec_tiles));
  p.G32 = static_cast<int>(cdiv(N, kNormGroup));
  size_t off = 0;
  p.off_err = off;
  off += 256;
  const size_t proj = align256(static_cast<size_t>(BH * N * D) * 2);
  const bool pp = variant == FLARE_VARIANT_FLAREPP || variant == FLARE_VARIANT_FLAREPP_OUT;
  if (pp) {
    p.off_kt = off; off += proj;
    p.off_vt = off; off += proj;
    p.off_kp = off; off += proj;
    p.off_vp = off; off += proj;
    p.off_kn_syn = off; off += align256(static_cast<size_t>(BH) * p.G32 * 4);
  }
  p.off_kn = off; off += align256(static_cast<size_t>(BH) * p.G32 * 4);
  p.off_part = off; off += align256(static_cast<size_t>(BH) * p.S * M * (D + 2) * 4);
  const size_t lat32 = align256(static_cast<size_t>(BH * M * D) * 4), lat16 = align256(static_cast<size_t>(BH * M * D) * 2);
  if (pp) {
    p.off_qx32 = off; off += lat32;
    p.off_qx16 = off; off += lat16;
  }
  p.off_z32 = off; off += lat32;
  p.off_z16 = off; off += lat16;
  p.off_fb = off; off += align256(static_cast<size_t>(BH) * N * 8);
  if (variant == FLARE_VARIANT_FLAREPP_OUT) {  // Y with the heads side by side, [B][N][C]
    p.off_ycat = off; off += proj;
  }
  p.total = off;
  return p;
}

// Workspace of the backward: the forward's (projection outputs, error word)
// followed by the fp32 recompute and gradient buffers.
struct BwdPlan {
  Plan fwd;
  int S = 1, tps = 1, rpb = 32, LB = 1, dw_splits = 1;
  size_t off_q32 = 0, off_qx32 = 0, off_lsyn = 0, off_dqx32 = 0, off_gsyn = 0, off_z32 = 0, off_lenc = 0,
         off_ltok = 0, off_dtok = 0, off_dz32 = 0, off_gam = 0, off_fpart = 0, off_pa = 0, off_pc = 0,
         off_g32 = 0, off_dwpart = 0, off_qpad = 0, off_q0pad = 0, off_zpad = 0, off_dzpad = 0, off_dqxpad = 0,
         off_dqxdec = 0, total = 0;
};

BwdPlan make_bwd_plan(bool pp, long B, long H, long N, long M, long D, long C) {
  BwdPlan bp;
  bp.fwd = make_plan(pp ? FLARE_VARIANT_FLAREPP : FLARE_VARIANT_FLARE, B, H, N, M, D);
  const long BH = B * H;
  // latent-parallel passes: 32, 64, 96 or 128 latent rows per CTA, so that
  // both a warp per 16 rows and a warp per 32 rows give whole warps
  bp.rpb = static_cast<int>(std::min(128L, cdiv(M, 32) * 32));
  bp.LB = static_cast<int>(cdiv(M, bp.rpb));
  // token splits: whole waves of CTAs (about 128 registers per thread, so
  // 256 / rows_per_block CTAs per SM), by the encoder's cost model
  const long ntiles = cdiv(N, kBwdTokTile);
  bp.S = choose_splits(BH * bp.LB, ntiles, static_cast<long>(kNumSM) * std::max(1, 256 / bp.rpb));
  bp.tps = static_cast<int>(cdiv(ntiles, bp.S));
  bp.S = static_cast<int>(cdiv(ntiles, bp.tps));
  bp.dw_splits = static_cast<int>(cdiv(B * N, kBwdDwRows));
  size_t off = bp.fwd.total;
  auto take = [&off](size_t bytes) {
    const size_t o = off;
    off += align256(bytes);
    return o;
  };
  const size_t lat = static_cast<size_t>(BH * M * D) * 4, row = static_cast<size_t>(BH * M) * 4;
  const size_t tokv = static_cast<size_t>(BH * N) * 4;
  const size_t part = static_cast<size_t>(BH) * bp.S * M * D * 4;
  bp.off_q32 = take(static_cast<size_t>(H * M * D) * 4);
  if (pp) {
    bp.off_qx32 = take(lat);
    bp.off_lsyn = take(row);
    bp.off_dqx32 = take(lat);
    bp.off_gsyn = take(row);
  }
  bp.off_z32 = take(lat);
  bp.off_lenc = take(row);
  bp.off_ltok = take(tokv);
  bp.off_dtok = take(tokv);
  bp.off_dz32 = take(lat);
  bp.off_gam = take(row);
  bp.off_fpart = take(static_cast<size_t>(BH) * bp.S * M * (D + 2) * 4);
  bp.off_pa = take(2 * part);  // [dZ partials | dQ partials] of the decoder backward
  bp.off_pc = take(part);
  // padded tf32 images ([rows][D + 4]) read by the token-parallel pass
  const size_t padded = static_cast<size_t>(BH * M * (D + 4)) * 4;
  bp.off_qpad = take(padded);
  bp.off_zpad = take(padded);
  bp.off_dzpad = take(padded);
  if (pp) {
    bp.off_q0pad = take(static_cast<size_t>(H * M * (D + 4)) * 4);
    bp.off_dqxpad = take(padded);
    bp.off_dqxdec = take(lat);
  }
  if (pp) {
    bp.off_g32 = take(static_cast<size_t>(B * N) * 4 * C * 4);
    bp.off_dwpart = take(static_cast<size_t>(bp.dw_splits) * C * 4 * C * 4);
  }
  bp.total = off;
  return bp;
}

// Records stage event i (a cudaEvent_t passed as void*) when profiling is on.
bool record(void* const* ev, int i, cudaStream_t s) {
  if (ev == nullptr || ev[i] == nullptr) return true;
  return cudaEventRecord(static_cast<cudaEvent_t>(ev[i]), s) == cudaSuccess;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

flare_status check_common(int B, int H, int N, int M, int D) {
  if (B < 1 || H < 1 || N < 1 || M < 1 || D < 1) return FLARE_ERR_SHAPE;
  if (D != 16 && D != 32) return FLARE_ERR_UNSUPPORTED;
  if (M % 16 != 0 || M > 512) return FLARE_ERR_UNSUPPORTED;
  // element offsets stay below 2^31 per head row index; whole tensors may be larger
  if (static_cast<long>(N) * D >= (1L << 31) || static_cast<long>(B) * H > (1L << 20)) return FLARE_ERR_UNSUPPORTED;
  return FLARE_OK;
}

float resolve_scale(float scale, int D) { return scale > 0.f ? scale : 1.0f / std::sqrt(static_cast<float>(D)); }

// Encoder pass: split partials of queries (bf16, [G][M][D]) against the keys
// and values of one shard ([B*H][N][D]; tokens [tok_offset, tok_offset + N) of
// sequences of n_global tokens) into part ([B*H][S][M][D+2] fp32).
flare_status run_encode_partials(const Plan& pl, uint8_t* ws, const void* q, int q_per_batch, const void* k,
                                 const void* v, const float* knorm, float* part, int B, int H, int N, int M, int D,
                                 const int32_t* lengths, int tok_offset, int n_global, float scale, cudaStream_t st,
                                 void* const* ev, int ev0) {
  const long BH = static_cast<long>(B) * H;
  const long G = q_per_batch ? BH : H;
  CUtensorMap tq, tk, tv;
  if (!map3d(&tq, q, D, M, G, D, std::min(M, kLatBlock), row_swizzle(D)) ||
      !map3d(&tk, k, D, N, BH, D, enc_tile(D), row_swizzle(D)) || !map3d(&tv, v, D, N, BH, D, enc_tile(D), row_swizzle(D)))
    return FLARE_ERR_LAUNCH;
  EncodeParams ep{};
  ep.B = B; ep.H = H; ep.N = N; ep.M = M; ep.D = D;
  ep.q_per_batch = q_per_batch;
  ep.n_splits = pl.S; ep.tiles_per_split = pl.tps; ep.n_lblocks = pl.LB; ep.n_groups32 = pl.G32;
  ep.q_rows = std::min(M, kLatBlock);
  ep.tok_offset = tok_offset; ep.n_global = n_global;
  ep.c = scale * 1.4426950408889634f;
  ep.lengths = lengths;
  ep.knorm = knorm;
  ep.q = static_cast<const uint16_t*>(q);
  ep.part = part;
  ep.err = reinterpret_cast<uint32_t*>(ws + pl.off_err);
  ep.timeout_ns = wait_timeout_ns();
  if (launch_encode(tq, tk, tv, ep, st) != cudaSuccess || !record(ev, ev0, st)) return FLARE_ERR_LAUNCH;
  return FLARE_OK;
}

// Merge of the partials of R shards ([R][B*H][S][M][D+2], rank-major) into
// out32/out16 ([B*H][M][D]).  With R == 1, q/k/v serve the exact
// recomputation of rows whose sums underflowed.
flare_status run_merge(const Plan& pl, uint8_t* ws, const float* part, int R, const void* q, int q_per_batch,
                       const void* k, const void* v, float* out32, uint16_t* out16, int B, int H, int N, int M,
                       int D, const int32_t* lengths, float scale, cudaStream_t st, void* const* ev, int ev_i,
                       bool allow_exact = true) {
  MergeParams mp{};
  mp.B = B; mp.H = H; mp.N = N; mp.M = M; mp.D = D;
  mp.q_per_batch = q_per_batch;
  mp.n_splits = pl.S; mp.tiles_per_split = pl.tps;
  mp.n_ranks = R;
  mp.allow_exact = allow_exact ? 1 : 0;
  mp.rank_stride = static_cast<size_t>(B) * H * pl.S * M * (D + 2);
  mp.err = reinterpret_cast<uint32_t*>(ws + pl.off_err);
  mp.scale = scale; mp.c = scale * 1.4426950408889634f;
  mp.lengths = lengths;
  mp.part = part;
  mp.q = static_cast<const uint16_t*>(q);
  mp.k = static_cast<const uint16_t*>(k);
  mp.v = static_cast<const uint16_t*>(v);
  mp.out_f32 = out32;
  mp.out_bf16 = out16;
  if (launch_merge(mp, st) != cudaSuccess || !record(ev, ev_i, st)) return FLARE_ERR_LAUNCH;
  return FLARE_OK;
}

// Encoder pass + merge on one GPU (the whole sequence).
flare_status run_encode(const Plan& pl, uint8_t* ws, const void* q, int q_per_batch, const void* k, const void* v,
                        const float* knorm, float* out32, uint16_t* out16, int B, int H, int N, int M, int D,
                        const int32_t* lengths, float scale, cudaStream_t st, void* const* ev, int ev0) {
  float* part = reinterpret_cast<float*>(ws + pl.off_part);
  flare_status r = run_encode_partials(pl, ws, q, q_per_batch, k, v, knorm, part, B, H, N, M, D, lengths, 0, N,
                                       scale, st, ev, ev0);
  if (r != FLARE_OK) return r;
  return run_merge(pl, ws, part, 1, q, q_per_batch, k, v, out32, out16, B, H, N, M, D, lengths, scale, st, ev,
                   ev0 + 1);
}

flare_status run_decode(const Plan& pl, uint8_t* ws, const void* q, int q_per_batch, const uint16_t* z16,
                        const void* k, void* y, int y_token_major, int B, int H, int N, int M, int D,
                        const int32_t* lengths, float scale, cudaStream_t st, int tok_offset = 0,
                        int n_global = -1) {
  const long BH = static_cast<long>(B) * H;
  const long G = q_per_batch ? BH : H;
  CUtensorMap tq, tz, tk;
  const int box_rows = std::min(M, 256);
  if (!map3d(&tq, q, D, M, G, D, box_rows, row_swizzle(D)) || !map3d(&tz, z16, D, M, BH, D, box_rows, row_swizzle(D)) ||
      !map3d(&tk, k, D, N, BH, D, kDecTile, row_swizzle(D)))
    return FLARE_ERR_LAUNCH;
  DecodeParams dp{};
  dp.B = B; dp.H = H; dp.N = N; dp.M = M; dp.D = D;
  dp.q_per_batch = q_per_batch;
  dp.tiles_per_cta = pl.dec_tiles; dp.ctas_per_head = pl.dec_ctas;
  dp.qz_box_rows = box_rows;
  dp.scale = scale; dp.c = scale * 1.4426950408889634f;
  dp.lengths = lengths;
  dp.q = static_cast<const uint16_t*>(q);
  dp.z = z16;
  dp.k = static_cast<const uint16_t*>(k);
  dp.y = static_cast<uint16_t*>(y);
  dp.y_token_major = y_token_major;
  dp.tok_offset = tok_offset;
  dp.n_global = n_global < 0 ? N : n_global;
  dp.err = reinterpret_cast<uint32_t*>(ws + pl.off_err);
  dp.fb_count = reinterpret_cast<uint32_t*>(ws + pl.off_err) + 1;
  dp.fb_list = reinterpret_cast<uint64_t*>(ws + pl.off_fb);
  dp.timeout_ns = wait_timeout_ns();
  if (launch_decode(tq, tz, tk, dp, st) != cudaSuccess) return FLARE_ERR_LAUNCH;
  return FLARE_OK;
}

}  // namespace
}  // namespace flare

namespace flare {
namespace {

// Scratch for callers that cannot allocate device memory (see
// flare_mixer_fwd_static): a fixed array in the library's device image.
// Every device that loads the library holds it until the process exits.
static __device__ __align__(256) unsigned char g_static_scratch[FLARE_STATIC_SCRATCH_BYTES];

// Device address of g_static_scratch on the current device.  Host code must
// not pass the symbol itself to a kernel (on the host it is only a stand-in);
// its device address is looked up once per device, with that device current.
flare_status static_scratch_address(void** out) {
  static std::mutex mu;
  static void* addr[256] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 256) return FLARE_ERR_LAUNCH;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) return FLARE_ERR_LAUNCH;
    addr[dev] = p;
  }
  *out = addr[dev];
  return FLARE_OK;
}

}  // namespace
}  // namespace flare

using namespace flare;

extern "C" {

size_t flare_workspace_bytes(int variant, int B, int H, int N, int M, int D, int C) {
  if (variant < FLARE_VARIANT_FLARE || variant > FLARE_VARIANT_FLAREPP_BWD) return 0;
  if (check_common(B, H, N, M, D) != FLARE_OK) return 0;
  const bool pp = variant != FLARE_VARIANT_FLARE && variant != FLARE_VARIANT_FLARE_BWD;
  if (pp && (C != H * D || C % 64 != 0 || C > 256)) return 0;
  if (variant == FLARE_VARIANT_FLARE_BWD || variant == FLARE_VARIANT_FLAREPP_BWD) {
    if (static_cast<long>(B) * H > 65535) return 0;
    return make_bwd_plan(pp, B, H, N, M, D, C).total;
  }
  return make_plan(variant, B, H, N, M, D).total;
}

const char* flare_status_string(flare_status s) {
  switch (s) {
    case FLARE_OK: return "FLARE_OK";
    case FLARE_ERR_NULL: return "FLARE_ERR_NULL: a required pointer is NULL";
    case FLARE_ERR_SHAPE: return "FLARE_ERR_SHAPE: a size is out of range or inconsistent";
    case FLARE_ERR_UNSUPPORTED: return "FLARE_ERR_UNSUPPORTED: size not covered by this build";
    case FLARE_ERR_ALIGN: return "FLARE_ERR_ALIGN: pointer not 16-byte (workspace 256-byte) aligned";
    case FLARE_ERR_WORKSPACE: return "FLARE_ERR_WORKSPACE: workspace too small";
    case FLARE_ERR_LAUNCH: return "FLARE_ERR_LAUNCH: CUDA error while enqueueing";
    case FLARE_ERR_TIMEOUT: return "FLARE_ERR_TIMEOUT: a device-side bounded wait expired";
    case FLARE_ERR_UNDERFLOW:
      return "FLARE_ERR_UNDERFLOW: a context-parallel merge found sums that underflowed (not recomputed)";
  }
  return "unknown flare_status";
}

flare_status flare_mixer_fwd_profiled(const flare_bf16* K, const flare_bf16* V, const flare_bf16* Q, flare_bf16* Y,
                                      int B, int H, int N, int M, int D, const int32_t* lengths, float scale,
                                      void* workspace, size_t workspace_bytes, void* stream, float* Z_out,
                                      void* const* stage_events) {
  if (!K || !V || !Q || !Y || !workspace) return FLARE_ERR_NULL;
  flare_status st = check_common(B, H, N, M, D);
  if (st != FLARE_OK) return st;
  if (!aligned16(K) || !aligned16(V) || !aligned16(Q) || !aligned16(Y) || !aligned16(lengths) || !aligned16(Z_out) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return FLARE_ERR_ALIGN;
  const Plan pl = make_plan(FLARE_VARIANT_FLARE, B, H, N, M, D);
  if (workspace_bytes < pl.total) return FLARE_ERR_WORKSPACE;
  const float sc = resolve_scale(scale, D);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  if (cudaMemsetAsync(ws + pl.off_err, 0, 8, s) != cudaSuccess) return FLARE_ERR_LAUNCH;
  if (!record(stage_events, 0, s)) return FLARE_ERR_LAUNCH;
  KnormParams kp{B * H, N, D, pl.G32, reinterpret_cast<const uint16_t*>(K), reinterpret_cast<float*>(ws + pl.off_kn)};
  if (launch_knorm(kp, s) != cudaSuccess || !record(stage_events, 1, s)) return FLARE_ERR_LAUNCH;
  float* z32 = Z_out ? Z_out : reinterpret_cast<float*>(ws + pl.off_z32);
  uint16_t* z16 = reinterpret_cast<uint16_t*>(ws + pl.off_z16);
  st = run_encode(pl, ws, Q, 0, K, V, kp.knorm, z32, z16, B, H, N, M, D, lengths, sc, s, stage_events, 2);
  if (st != FLARE_OK) return st;
  st = run_decode(pl, ws, Q, 0, z16, K, Y, 0, B, H, N, M, D, lengths, sc, s);
  if (st != FLARE_OK) return st;
  return record(stage_events, 4, s) ? FLARE_OK : FLARE_ERR_LAUNCH;
}

flare_status flare_mixer_fwd(const flare_bf16* K, const flare_bf16* V, const flare_bf16* Q, flare_bf16* Y, int B,
                             int H, int N, int M, int D, const int32_t* lengths, float scale, void* workspace,
                             size_t workspace_bytes, void* stream, float* Z_out) {
  return flare_mixer_fwd_profiled(K, V, Q, Y, B, H, N, M, D, lengths, scale, workspace, workspace_bytes, stream,
                                  Z_out, nullptr);
}

}  // extern "C"

namespace flare {
namespace {

// Shape, pointer and alignment checks shared by the FLARE++ entry points.
flare_status check_flarepp(const void* X, const void* Wk, const void* Wv, const void* Wk_syn, const void* Wv_syn,
                           const void* Q0, const void* Y, int B, int N, int C, int H, int M, int D,
                           const int32_t* lengths, const void* workspace, const float* Qx_out, const float* Z_out) {
  if (!X || !Wk || !Wv || !Wk_syn || !Wv_syn || !Q0 || !Y || !workspace) return FLARE_ERR_NULL;
  flare_status st = check_common(B, H, N, M, D);
  if (st != FLARE_OK) return st;
  if (C != H * D) return FLARE_ERR_SHAPE;
  if (C % 64 != 0 || C > 256) return FLARE_ERR_UNSUPPORTED;
  if (!aligned16(X) || !aligned16(Wk) || !aligned16(Wv) || !aligned16(Wk_syn) || !aligned16(Wv_syn) ||
      !aligned16(Q0) || !aligned16(Y) || !aligned16(lengths) || !aligned16(Qx_out) || !aligned16(Z_out) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return FLARE_ERR_ALIGN;
  return FLARE_OK;
}

// Projection launch: n_proj weights (tensor maps tw[0..n_proj)) into out[]
// ([B][H][N][D], or [B][N][C] when token_major), key norms where given.
flare_status run_project(const Plan& pl, uint8_t* ws, const CUtensorMap& tx, const CUtensorMap (&tw)[4], int n_proj,
                         int token_major, uint16_t* const (&out)[4], float* const (&knorm)[4], int B, int N, int C,
                         int H, int D, cudaStream_t s) {
  ProjParams pp{};
  pp.B = B; pp.N = N; pp.C = C; pp.H = H; pp.D = D;
  pp.tiles_per_b = static_cast<int>(cdiv(N, kProjTile));
  pp.n_tiles = B * pp.tiles_per_b;
  const int slots = C == 256 ? kNumSM : kNumSM * 2;
  pp.groups = std::max(1, std::min(pp.n_tiles, slots / n_proj));
  pp.n_groups32 = pl.G32;
  pp.n_proj = n_proj;
  pp.token_major = token_major;
  for (int i = 0; i < 4; ++i) {
    pp.out[i] = out[i];
    pp.knorm[i] = knorm[i];
  }
  pp.err = reinterpret_cast<uint32_t*>(ws + pl.off_err);
  pp.timeout_ns = wait_timeout_ns();
  return launch_project(tx, tw, pp, s) == cudaSuccess ? FLARE_OK : FLARE_ERR_LAUNCH;
}

// Outputs of the FLARE++ projections in the workspace.
struct Projected {
  uint16_t *kt, *vt, *kk, *vv;
  float *kn_syn, *kn;
};

// eq. 7 and eq. 9: the per-head projections of X (two when the synthesis
// and encode weights are the same tensors, else four).
flare_status flarepp_project(const Plan& pl, const flare_bf16* X, const flare_bf16* Wk, const flare_bf16* Wv,
                             const flare_bf16* Wk_syn, const flare_bf16* Wv_syn, int B, int N, int C, int H, int D,
                             uint8_t* ws, cudaStream_t s, void* const* stage_events, Projected* pr) {
  // The same weights for synthesis and encode (the shared-projection
  // variant): K~ = K and V~ = V, so two projections serve both passes.
  const bool shared = Wk_syn == Wk && Wv_syn == Wv;
  // eq. 7 and eq. 9: the per-head projections
  CUtensorMap tx, tw[4];
  const flare_bf16* w[4] = {Wk_syn, Wv_syn, Wk, Wv};
  if (shared) {
    w[0] = Wk;
    w[1] = Wv;
  }
  if (!map3d(&tx, X, C, N, B, 64, kProjTile, CU_TENSOR_MAP_SWIZZLE_128B)) return FLARE_ERR_LAUNCH;
  for (int i = 0; i < 4; ++i)
    if (!map2d(&tw[i], w[i], C, C, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B)) return FLARE_ERR_LAUNCH;
  uint16_t* kt = reinterpret_cast<uint16_t*>(ws + pl.off_kt);
  uint16_t* vt = reinterpret_cast<uint16_t*>(ws + pl.off_vt);
  uint16_t* kk = reinterpret_cast<uint16_t*>(ws + pl.off_kp);
  uint16_t* vv = reinterpret_cast<uint16_t*>(ws + pl.off_vp);
  float* kn_syn = reinterpret_cast<float*>(ws + pl.off_kn_syn);
  float* kn = reinterpret_cast<float*>(ws + pl.off_kn);
  if (shared) {
    kt = kk;
    vt = vv;
    kn_syn = kn;
  }
  if (!record(stage_events, 0, s)) return FLARE_ERR_LAUNCH;
  uint16_t* const outs[4] = {kt, vt, kk, vv};
  float* const norms[4] = {kn_syn, nullptr, kn, nullptr};
  flare_status st = run_project(pl, ws, tx, tw, shared ? 2 : 4, 0, outs, norms, B, N, C, H, D, s);
  if (st != FLARE_OK || !record(stage_events, 1, s)) return FLARE_ERR_LAUNCH;
  *pr = Projected{kt, vt, kk, vv, kn_syn, kn};
  return FLARE_OK;
}

// The FLARE++ pipeline (eq. 7-11) after the argument checks.  Y is written
// [B][H][N][D], or [B][N][C] when y_token_major.
flare_status flarepp_run(const Plan& pl, const flare_bf16* X, const flare_bf16* Wk, const flare_bf16* Wv,
                         const flare_bf16* Wk_syn, const flare_bf16* Wv_syn, const flare_bf16* Q0, void* Y,
                         int y_token_major, int B, int N, int C, int H, int M, int D, const int32_t* lengths,
                         float sc, uint8_t* ws, cudaStream_t s, float* Qx_out, float* Z_out,
                         void* const* stage_events) {
  if (cudaMemsetAsync(ws + pl.off_err, 0, 8, s) != cudaSuccess) return FLARE_ERR_LAUNCH;
  Projected pr;
  flare_status st = flarepp_project(pl, X, Wk, Wv, Wk_syn, Wv_syn, B, N, C, H, D, ws, s, stage_events, &pr);
  if (st != FLARE_OK) return st;
  uint16_t *kt = pr.kt, *vt = pr.vt, *kk = pr.kk, *vv = pr.vv;
  float *kn_syn = pr.kn_syn, *kn = pr.kn;

  // eq. 8: query synthesis with the learned seeds
  float* qx32 = Qx_out ? Qx_out : reinterpret_cast<float*>(ws + pl.off_qx32);
  uint16_t* qx16 = reinterpret_cast<uint16_t*>(ws + pl.off_qx16);
  st = run_encode(pl, ws, Q0, 0, kt, vt, kn_syn, qx32, qx16, B, H, N, M, D, lengths, sc, s, stage_events, 2);
  if (st != FLARE_OK) return st;
  // eq. 10: encode with the synthesised queries
  float* z32 = Z_out ? Z_out : reinterpret_cast<float*>(ws + pl.off_z32);
  uint16_t* z16 = reinterpret_cast<uint16_t*>(ws + pl.off_z16);
  st = run_encode(pl, ws, qx16, 1, kk, vv, kn, z32, z16, B, H, N, M, D, lengths, sc, s, stage_events, 4);
  if (st != FLARE_OK) return st;
  // eq. 11: decode
  st = run_decode(pl, ws, qx16, 1, z16, kk, Y, y_token_major, B, H, N, M, D, lengths, sc, s);
  if (st != FLARE_OK) return st;
  return record(stage_events, 6, s) ? FLARE_OK : FLARE_ERR_LAUNCH;
}

}  // namespace
}  // namespace flare

extern "C" {

flare_status flarepp_mixer_fwd_profiled(const flare_bf16* X, const flare_bf16* Wk, const flare_bf16* Wv,
                                        const flare_bf16* Wk_syn, const flare_bf16* Wv_syn, const flare_bf16* Q0,
                                        flare_bf16* Y, int B, int N, int C, int H, int M, int D,
                                        const int32_t* lengths, float scale, void* workspace,
                                        size_t workspace_bytes, void* stream, float* Qx_out, float* Z_out,
                                        void* const* stage_events) {
  flare_status st = check_flarepp(X, Wk, Wv, Wk_syn, Wv_syn, Q0, Y, B, N, C, H, M, D, lengths, workspace, Qx_out,
                                  Z_out);
  if (st != FLARE_OK) return st;
  const Plan pl = make_plan(FLARE_VARIANT_FLAREPP, B, H, N, M, D);
  if (workspace_bytes < pl.total) return FLARE_ERR_WORKSPACE;
  return flarepp_run(pl, X, Wk, Wv, Wk_syn, Wv_syn, Q0, Y, 0, B, N, C, H, M, D, lengths, resolve_scale(scale, D),
                     static_cast<uint8_t*>(workspace), static_cast<cudaStream_t>(stream), Qx_out, Z_out,
                     stage_events);
}

flare_status flarepp_mixer_out_fwd(const flare_bf16* X, const flare_bf16* Wk, const flare_bf16* Wv,
                                   const flare_bf16* Wk_syn, const flare_bf16* Wv_syn, const flare_bf16* Q0,
                                   const flare_bf16* Wo, flare_bf16* Out, int B, int N, int C, int H, int M, int D,
                                   const int32_t* lengths, float scale, void* workspace, size_t workspace_bytes,
                                   void* stream) {
  if (!Wo) return FLARE_ERR_NULL;
  flare_status st = check_flarepp(X, Wk, Wv, Wk_syn, Wv_syn, Q0, Out, B, N, C, H, M, D, lengths, workspace,
                                  nullptr, nullptr);
  if (st != FLARE_OK) return st;
  if (!aligned16(Wo)) return FLARE_ERR_ALIGN;
  const Plan pl = make_plan(FLARE_VARIANT_FLAREPP_OUT, B, H, N, M, D);
  if (workspace_bytes < pl.total) return FLARE_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint16_t* ycat = reinterpret_cast<uint16_t*>(ws + pl.off_ycat);  // [B][N][C], heads side by side
  st = flarepp_run(pl, X, Wk, Wv, Wk_syn, Wv_syn, Q0, ycat, 1, B, N, C, H, M, D, lengths, resolve_scale(scale, D),
                   ws, s, nullptr, nullptr, nullptr);
  if (st != FLARE_OK) return st;
  // Out = concat_h(Y_h) W_O: the same tcgen05 projection with one weight and
  // token-major output rows
  CUtensorMap ty, two[4];
  if (!map3d(&ty, ycat, C, N, B, 64, kProjTile, CU_TENSOR_MAP_SWIZZLE_128B)) return FLARE_ERR_LAUNCH;
  for (int i = 0; i < 4; ++i)
    if (!map2d(&two[i], Wo, C, C, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B)) return FLARE_ERR_LAUNCH;
  uint16_t* const outs[4] = {Out, nullptr, nullptr, nullptr};
  float* const norms[4] = {nullptr, nullptr, nullptr, nullptr};
  return run_project(pl, ws, ty, two, 1, 1, outs, norms, B, N, C, H, D, s);
}

flare_status flarepp_mixer_fwd(const flare_bf16* X, const flare_bf16* Wk, const flare_bf16* Wv,
                               const flare_bf16* Wk_syn, const flare_bf16* Wv_syn, const flare_bf16* Q0,
                               flare_bf16* Y, int B, int N, int C, int H, int M, int D, const int32_t* lengths,
                               float scale, void* workspace, size_t workspace_bytes, void* stream, float* Qx_out,
                               float* Z_out) {
  return flarepp_mixer_fwd_profiled(X, Wk, Wv, Wk_syn, Wv_syn, Q0, Y, B, N, C, H, M, D, lengths, scale, workspace,
                                    workspace_bytes, stream, Qx_out, Z_out, nullptr);
}

// ---------------------------------------------------------------------------
// Context parallelism (eq. 13-14): phases of one rank over its token shard
// ---------------------------------------------------------------------------

size_t flare_cp_partials_bytes(int B, int H, int N, int M, int D) {
  if (check_common(B, H, N, M, D) != FLARE_OK) return 0;
  const Plan pl = make_plan(FLARE_VARIANT_FLARE, B, H, N, M, D);
  return static_cast<size_t>(B) * H * pl.S * M * (D + 2) * sizeof(float);
}

}  // extern "C"

namespace flare {
namespace {

flare_status check_cp(int N, int rank, int world, const void* part) {
  if (!part) return FLARE_ERR_NULL;
  if (world < 1 || rank < 0 || rank >= world) return FLARE_ERR_SHAPE;
  if (static_cast<long>(N) * world >= (1L << 31)) return FLARE_ERR_UNSUPPORTED;
  if (!aligned16(part)) return FLARE_ERR_ALIGN;
  return FLARE_OK;
}

}  // namespace
}  // namespace flare

extern "C" {

flare_status flarepp_cp_begin(const flare_bf16* X, const flare_bf16* Wk, const flare_bf16* Wv,
                              const flare_bf16* Wk_syn, const flare_bf16* Wv_syn, const flare_bf16* Q0, int B, int N,
                              int C, int H, int M, int D, const int32_t* lengths, int rank, int world, float scale,
                              void* workspace, size_t workspace_bytes, void* stream, float* partials) {
  flare_status st = check_flarepp(X, Wk, Wv, Wk_syn, Wv_syn, Q0, X, B, N, C, H, M, D, lengths, workspace, nullptr,
                                  nullptr);
  if (st != FLARE_OK) return st;
  if ((st = check_cp(N, rank, world, partials)) != FLARE_OK) return st;
  const Plan pl = make_plan(FLARE_VARIANT_FLAREPP, B, H, N, M, D);
  if (workspace_bytes < pl.total) return FLARE_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(ws + pl.off_err, 0, 8, s) != cudaSuccess) return FLARE_ERR_LAUNCH;
  Projected pr;
  if ((st = flarepp_project(pl, X, Wk, Wv, Wk_syn, Wv_syn, B, N, C, H, D, ws, s, nullptr, &pr)) != FLARE_OK)
    return st;
  // eq. 8 on the local shard: the synthesis partials
  return run_encode_partials(pl, ws, Q0, 0, pr.kt, pr.vt, pr.kn_syn, partials, B, H, N, M, D, lengths, rank * N,
                             world * N, resolve_scale(scale, D), s, nullptr, 0);
}

flare_status flarepp_cp_middle(const float* partials_all, int B, int N, int C, int H, int M, int D,
                               const int32_t* lengths, int rank, int world, float scale, void* workspace,
                               size_t workspace_bytes, void* stream, float* partials, float* Qx_out) {
  if (!partials_all || !workspace) return FLARE_ERR_NULL;
  flare_status st = check_common(B, H, N, M, D);
  if (st != FLARE_OK) return st;
  if (C != H * D || C % 64 != 0 || C > 256) return C != H * D ? FLARE_ERR_SHAPE : FLARE_ERR_UNSUPPORTED;
  if ((st = check_cp(N, rank, world, partials)) != FLARE_OK) return st;
  if (!aligned16(partials_all) || !aligned16(lengths) || !aligned16(Qx_out)) return FLARE_ERR_ALIGN;
  const Plan pl = make_plan(FLARE_VARIANT_FLAREPP, B, H, N, M, D);
  if (workspace_bytes < pl.total) return FLARE_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const float sc = resolve_scale(scale, D);
  float* qx32 = Qx_out ? Qx_out : reinterpret_cast<float*>(ws + pl.off_qx32);
  uint16_t* qx16 = reinterpret_cast<uint16_t*>(ws + pl.off_qx16);
  // Q(X): every rank merges the same partials in the same order
  st = run_merge(pl, ws, partials_all, world, nullptr, 0, nullptr, nullptr, qx32, qx16, B, H, N, M, D, lengths, sc, s,
                 nullptr, 0, false);
  if (st != FLARE_OK) return st;
  // eq. 10 on the local shard: the encode partials
  return run_encode_partials(pl, ws, qx16, 1, ws + pl.off_kp, ws + pl.off_vp, reinterpret_cast<float*>(ws + pl.off_kn),
                             partials, B, H, N, M, D, lengths, rank * N, world * N, sc, s, nullptr, 0);
}

flare_status flarepp_cp_end(const float* partials_all, flare_bf16* Y, int B, int N, int C, int H, int M, int D,
                            const int32_t* lengths, int rank, int world, float scale, void* workspace,
                            size_t workspace_bytes, void* stream, float* Z_out) {
  if (!partials_all || !Y || !workspace) return FLARE_ERR_NULL;
  flare_status st = check_common(B, H, N, M, D);
  if (st != FLARE_OK) return st;
  if (C != H * D || C % 64 != 0 || C > 256) return C != H * D ? FLARE_ERR_SHAPE : FLARE_ERR_UNSUPPORTED;
  if ((st = check_cp(N, rank, world, partials_all)) != FLARE_OK) return st;
  if (!aligned16(Y) || !aligned16(lengths) || !aligned16(Z_out)) return FLARE_ERR_ALIGN;
  const Plan pl = make_plan(FLARE_VARIANT_FLAREPP, B, H, N, M, D);
  if (workspace_bytes < pl.total) return FLARE_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const float sc = resolve_scale(scale, D);
  float* z32 = Z_out ? Z_out : reinterpret_cast<float*>(ws + pl.off_z32);
  uint16_t* z16 = reinterpret_cast<uint16_t*>(ws + pl.off_z16);
  st = run_merge(pl, ws, partials_all, world, nullptr, 0, nullptr, nullptr, z32, z16, B, H, N, M, D, lengths, sc, s,
                 nullptr, 0, false);
  if (st != FLARE_OK) return st;
  // eq. 11 on the local shard
  return run_decode(pl, ws, ws + pl.off_qx16, 1, z16, ws + pl.off_kp, Y, 0, B, H, N, M, D, lengths, sc, s, rank * N,
                    world * N);
}

flare_status flare_cp_begin(const flare_bf16* K, const flare_bf16* V, const flare_bf16* Q, int B, int H, int N, int M,
                            int D, const int32_t* lengths, int rank, int world, float scale, void* workspace,
                            size_t workspace_bytes, void* stream, float* partials) {
  if (!K || !V || !Q || !workspace) return FLARE_ERR_NULL;
  flare_status st = check_common(B, H, N, M, D);
  if (st != FLARE_OK) return st;
  if ((st = check_cp(N, rank, world, partials)) != FLARE_OK) return st;
  if (!aligned16(K) || !aligned16(V) || !aligned16(Q) || !aligned16(lengths) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return FLARE_ERR_ALIGN;
  const Plan pl = make_plan(FLARE_VARIANT_FLARE, B, H, N, M, D);
  if (workspace_bytes < pl.total) return FLARE_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(ws + pl.off_err, 0, 8, s) != cudaSuccess) return FLARE_ERR_LAUNCH;
  KnormParams kp{B * H, N, D, pl.G32, reinterpret_cast<const uint16_t*>(K), reinterpret_cast<float*>(ws + pl.off_kn)};
  if (launch_knorm(kp, s) != cudaSuccess) return FLARE_ERR_LAUNCH;
  return run_encode_partials(pl, ws, Q, 0, K, V, kp.knorm, partials, B, H, N, M, D, lengths, rank * N, world * N,
                             resolve_scale(scale, D), s, nullptr, 0);
}

flare_status flare_cp_end(const float* partials_all, const flare_bf16* K, const flare_bf16* Q, flare_bf16* Y, int B,
                          int H, int N, int M, int D, const int32_t* lengths, int rank, int world, float scale,
                          void* workspace, size_t workspace_bytes, void* stream, float* Z_out) {
  if (!partials_all || !K || !Q || !Y || !workspace) return FLARE_ERR_NULL;
  flare_status st = check_common(B, H, N, M, D);
  if (st != FLARE_OK) return st;
  if ((st = check_cp(N, rank, world, partials_all)) != FLARE_OK) return st;
  if (!aligned16(K) || !aligned16(Q) || !aligned16(Y) || !aligned16(lengths) || !aligned16(Z_out)) return FLARE_ERR_ALIGN;
  const Plan pl = make_plan(FLARE_VARIANT_FLARE, B, H, N, M, D);
  if (workspace_bytes < pl.total) return FLARE_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const float sc = resolve_scale(scale, D);
  float* z32 = Z_out ? Z_out : reinterpret_cast<float*>(ws + pl.off_z32);
  uint16_t* z16 = reinterpret_cast<uint16_t*>(ws + pl.off_z16);
  st = run_merge(pl, ws, partials_all, world, nullptr, 0, nullptr, nullptr, z32, z16, B, H, N, M, D, lengths, sc, s,
                 nullptr, 0, false);
  if (st != FLARE_OK) return st;
  return run_decode(pl, ws, Q, 0, z16, K, Y, 0, B, H, N, M, D, lengths, sc, s, rank * N, world * N);
}

flare_status flare_mixer_fwd_static(const flare_bf16* K, const flare_bf16* V, const flare_bf16* Q, flare_bf16* Y,
                                    int B, int H, int N, int M, int D, const int32_t* lengths, float scale,
                                    void* stream, float* Z_out) {
  // Same argument checks as flare_mixer_fwd, then the size limit of the
  // static scratch, all before any CUDA call.
  if (!K || !V || !Q || !Y) return FLARE_ERR_NULL;
  flare_status st = check_common(B, H, N, M, D);
  if (st != FLARE_OK) return st;
  if (!aligned16(K) || !aligned16(V) || !aligned16(Q) || !aligned16(Y) || !aligned16(lengths) || !aligned16(Z_out))
    return FLARE_ERR_ALIGN;
  if (make_plan(FLARE_VARIANT_FLARE, B, H, N, M, D).total > FLARE_STATIC_SCRATCH_BYTES) return FLARE_ERR_WORKSPACE;
  void* scratch = nullptr;
  st = static_scratch_address(&scratch);
  if (st != FLARE_OK) return st;
  return flare_mixer_fwd(K, V, Q, Y, B, H, N, M, D, lengths, scale, scratch, FLARE_STATIC_SCRATCH_BYTES, stream,
                         Z_out);
}

flare_status flare_last_device_status(void* workspace, void* stream) {
  if (!workspace) return FLARE_ERR_NULL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return FLARE_ERR_LAUNCH;
  uint32_t word = 0;
  if (cudaMemcpy(&word, workspace, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return FLARE_ERR_LAUNCH;
  if (word & FLARE_DEV_TIMEOUT) return FLARE_ERR_TIMEOUT;
  if (word & FLARE_DEV_BAD_LENGTH) return FLARE_ERR_SHAPE;
  if (word & FLARE_DEV_UNDERFLOW) return FLARE_ERR_UNDERFLOW;
  return FLARE_OK;
}

flare_status flare_selftest_wait_timeout(void* workspace, void* stream, unsigned long long timeout_ns) {
  if (!workspace) return FLARE_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return FLARE_ERR_ALIGN;
  if (timeout_ns < 1000ull) timeout_ns = 1000ull;
  if (timeout_ns > 1000000000ull) timeout_ns = 1000000000ull;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(workspace, 0, 4, s) != cudaSuccess) return FLARE_ERR_LAUNCH;
  if (launch_wait_selftest(static_cast<uint32_t*>(workspace), timeout_ns, s) != cudaSuccess) return FLARE_ERR_LAUNCH;
  return FLARE_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Backward (gradients)
// ---------------------------------------------------------------------------

namespace flare {
namespace {

constexpr float kLog2e = 1.4426950408889634f;

// Where the token-parallel pass writes dK and dV: token-major fp32 rows of
// the projection-gradient matrix, or bf16 [B][H][N][D] outputs.
struct TokOut {
  float* g32;
  int g_ld, col_k, col_v;
  uint16_t *dk16, *dv16;
};

// This GPU's token shard: tokens [tok_offset, tok_offset + N) of sequences
// of n_global tokens, one of R shards (R = 1: the whole sequence).
struct Shard {
  int tok_offset, n_global, R;
};

LatParams lat_params(const BwdPlan& bp, uint8_t* ws, const float* q, int q_per_batch, const void* k, int B, int H,
                     int N, int M, int D, const int32_t* lengths, float sc, const Shard& sh) {
  LatParams lp{};
  lp.B = B; lp.H = H; lp.N = N; lp.M = M; lp.D = D;
  lp.tok_offset = sh.tok_offset; lp.n_global = sh.n_global;
  lp.q_per_batch = q_per_batch;
  lp.n_splits = bp.S; lp.tiles_per_split = bp.tps; lp.rows_per_block = bp.rpb;
  lp.c = sc * kLog2e;
  lp.lengths = lengths;
  lp.q = q;
  lp.k = static_cast<const uint16_t*>(k);
  lp.err = reinterpret_cast<uint32_t*>(ws + bp.fwd.off_err);
  return lp;
}

TokParams tok_params(int B, int H, int N, int M, int D, int q_per_batch, const int32_t* lengths, float sc,
                     const Shard& sh) {
  TokParams tp{};
  tp.B = B; tp.H = H; tp.N = N; tp.M = M; tp.D = D;
  tp.tok_offset = sh.tok_offset; tp.n_global = sh.n_global;
  tp.q_per_batch = q_per_batch;
  tp.c = sc * kLog2e;
  tp.lengths = lengths;
  return tp;
}

// out = addend + mult * (sum over R shards and S splits of part0 (+ part1)),
// gamma = <out, zref> per row when zref is given.
flare_status lat_sum(int B, int H, int M, int D, int S, int fold_batch, float mult, const float* part0,
                     const float* part1, int R, size_t rank_stride, const float* addend, const float* zref,
                     float* gamma, float* out, cudaStream_t s) {
  LatSumParams p{};
  p.B = B; p.H = H; p.M = M; p.D = D; p.S = S;
  p.fold_batch = fold_batch; p.mult = mult;
  p.part0 = part0; p.part1 = part1; p.zref = zref; p.gamma = gamma; p.out = out;
  p.R = R; p.rank_stride = rank_stride; p.addend = addend;
  return launch_lat_sum(p, s) == cudaSuccess ? FLARE_OK : FLARE_ERR_LAUNCH;
}

// Merge of the recompute partials of R shards: Z (or Q(X)) and L_m.
flare_status lat_merge(const float* part, int R, size_t rank_stride, int BH, int M, int D, int S, float* z,
                       float* lse, cudaStream_t s) {
  LatMergeParams mp{};
  mp.BH = BH; mp.M = M; mp.D = D; mp.S = S;
  mp.R = R; mp.rank_stride = rank_stride;
  mp.part = part; mp.z = z; mp.lse = lse;
  return launch_lat_merge(mp, s) == cudaSuccess ? FLARE_OK : FLARE_ERR_LAUNCH;
}

flare_status pad(const float* src, float* dst, long rows, int D, float mul, cudaStream_t s) {
  const PadParams pp{rows, D, mul, src, dst};
  return launch_pad(pp, s) == cudaSuccess ? FLARE_OK : FLARE_ERR_LAUNCH;
}

// fp32 elements of one split-partials buffer [B*H][S][M][D] (+2 per row for
// the recompute partials).
size_t part_floats(const BwdPlan& bp, int B, int H, int M, int D, bool recompute) {
  return static_cast<size_t>(B) * H * bp.S * M * (D + (recompute ? 2 : 0));
}

// FLARE (eq. 5-6) backward on one GPU: dK, dV to bf16 outputs, dQ summed
// over the batch.
flare_status flare_bwd_run(const BwdPlan& bp, uint8_t* ws, const float* q, const void* k, const void* v,
                           const void* dy, uint16_t* dk, uint16_t* dv, float* dq, int B, int H, int N, int M, int D,
                           const int32_t* lengths, float sc, cudaStream_t s) {
  const Shard sh{0, N, 1};
  const long BH = static_cast<long>(B) * H;
  float* z32 = reinterpret_cast<float*>(ws + bp.off_z32);
  float* lenc = reinterpret_cast<float*>(ws + bp.off_lenc);
  float* dz32 = reinterpret_cast<float*>(ws + bp.off_dz32);
  float* gam = reinterpret_cast<float*>(ws + bp.off_gam);
  float* pa = reinterpret_cast<float*>(ws + bp.off_pa);
  float* pb = pa + part_floats(bp, B, H, M, D, false);
  float* pc = reinterpret_cast<float*>(ws + bp.off_pc);
  float* qpad = reinterpret_cast<float*>(ws + bp.off_qpad);
  float* zpad = reinterpret_cast<float*>(ws + bp.off_zpad);
  float* dzpad = reinterpret_cast<float*>(ws + bp.off_dzpad);
  // encoder recompute: Z and the row normalisers
  LatParams lf = lat_params(bp, ws, q, 0, k, B, H, N, M, D, lengths, sc, sh);
  lf.v = static_cast<const uint16_t*>(v);
  lf.part_a = reinterpret_cast<float*>(ws + bp.off_fpart);
  if (launch_lat(kLatForward, lf, s) != cudaSuccess) return FLARE_ERR_LAUNCH;
  flare_status st = lat_merge(lf.part_a, 1, 0, static_cast<int>(BH), M, D, bp.S, z32, lenc, s);
  if (st != FLARE_OK) return st;
  if ((st = pad(q, qpad, static_cast<long>(H) * M, D, sc * kLog2e, s)) != FLARE_OK ||
      (st = pad(z32, zpad, BH * M, D, 1.f, s)) != FLARE_OK)
    return st;
  // decoder recompute: L_n and delta_n
  TokParams tp = tok_params(B, H, N, M, D, 0, lengths, sc, sh);
  tp.qpad = qpad; tp.zpad = zpad; tp.dzpad = dzpad; tp.lm = lenc; tp.gam = gam;
  tp.k = static_cast<const uint16_t*>(k);
  tp.v = static_cast<const uint16_t*>(v);
  tp.dy = static_cast<const uint16_t*>(dy);
  tp.ltok = reinterpret_cast<float*>(ws + bp.off_ltok);
  tp.dtok = reinterpret_cast<float*>(ws + bp.off_dtok);
  tp.dk16 = dk; tp.dv16 = dv;
  if (launch_tok(kTokStats, tp, s) != cudaSuccess) return FLARE_ERR_LAUNCH;
  // decoder backward, reductions over tokens: dZ and the decoder's dQ
  LatParams ld = lat_params(bp, ws, q, 0, k, B, H, N, M, D, lengths, sc, sh);
  ld.zrow = z32; ld.dy = tp.dy; ld.ltok = tp.ltok; ld.dtok = tp.dtok;
  ld.part_a = pa; ld.part_b = pb;
  if (launch_lat(kLatDecoder, ld, s) != cudaSuccess) return FLARE_ERR_LAUNCH;
  if ((st = lat_sum(B, H, M, D, bp.S, 0, 1.f, pa, nullptr, 1, 0, nullptr, z32, gam, dz32, s)) != FLARE_OK ||
      (st = pad(dz32, dzpad, BH * M, D, 1.f, s)) != FLARE_OK)
    return st;
  // dK (both parts) and dV
  if (launch_tok(kTokFull, tp, s) != cudaSuccess) return FLARE_ERR_LAUNCH;
  // encoder backward: its dQ; dQ = scale * (decoder + encoder parts), summed over the batch
  LatParams le = lat_params(bp, ws, q, 0, k, B, H, N, M, D, lengths, sc, sh);
  le.zrow = dz32; le.lrow = lenc; le.grow = gam; le.v = tp.v;
  le.part_b = pc;
  if (launch_lat(kLatEncoder, le, s) != cudaSuccess) return FLARE_ERR_LAUNCH;
  return lat_sum(B, H, M, D, bp.S, 1, sc, pb, pc, 1, 0, nullptr, nullptr, nullptr, dq, s);
}

// ---------------------------------------------------------------------------
// FLARE++ (eq. 7-11) backward in seven phases.  Between two phases every
// shard's exchange buffer is all-gathered in rank order; the next phase reads
// the gathered buffers (R shards, `stride` floats apart) and merges them in
// ascending (rank, split) order, so every rank holds bitwise the same Q(X),
// Z, dZ, dQ(X), dQ0 and dW.  On one GPU the phases run back to back with the
// exchanges in the workspace.  The workspace carries the shard's state
// (projections, Q(X), Z, normalisers, gradient rows) from phase to phase.
//   0: projections; synthesis recompute partials                 -> E0
//   1: merge E0 -> Q(X), L~_m; encode recompute partials         -> E1
//   2: merge E1 -> Z, L_m; decoder stats; decoder backward       -> E2 = [dZ | dQ_dec partials]
//   3: dZ, gamma, scale * dQ_dec; dK, dV rows; encoder dQ        -> E3
//   4: dQ(X), gamma~; dK~, dV~ rows; synthesis dQ0 partials      -> E4
//   5: dQ0; dX (local rows); dW partials of the local rows       -> E5
//   6: dW
// ---------------------------------------------------------------------------
constexpr int kPpPhases = 7;

struct PpArgs {
  const flare_bf16 *X, *Wk, *Wv, *Wk_syn, *Wv_syn, *Q0, *dY;
  flare_bf16* dX;
  float *dWk, *dWv, *dWk_syn, *dWv_syn, *dQ0;
  int B, N, C, H, M, D;
  const int32_t* lengths;
  float sc;
  Shard sh;
};

size_t pp_exchange_floats(const BwdPlan& bp, int phase, int B, int H, int M, int D, int C) {
  switch (phase) {
    case 0:
    case 1: return part_floats(bp, B, H, M, D, true);
    case 2: return 2 * part_floats(bp, B, H, M, D, false);
    case 3:
    case 4: return part_floats(bp, B, H, M, D, false);
    case 5: return static_cast<size_t>(bp.dw_splits) * C * 4 * C;
    default: return 0;
  }
}

flare_status pp_phase(int phase, const BwdPlan& bp, uint8_t* ws, const PpArgs& a, const float* gathered,
                      float* exch, cudaStream_t s) {
  const int B = a.B, N = a.N, C = a.C, H = a.H, M = a.M, D = a.D;
  const long BH = static_cast<long>(B) * H;
  const float sc = a.sc, c = sc * kLog2e;
  const int R = a.sh.R;
  const bool shared = a.Wk_syn == a.Wk && a.Wv_syn == a.Wv;
  uint16_t* kk = reinterpret_cast<uint16_t*>(ws + bp.fwd.off_kp);
  uint16_t* vv = reinterpret_cast<uint16_t*>(ws + bp.fwd.off_vp);
  uint16_t* kt = shared ? kk : reinterpret_cast<uint16_t*>(ws + bp.fwd.off_kt);
  uint16_t* vt = shared ? vv : reinterpret_cast<uint16_t*>(ws + bp.fwd.off_vt);
  float* q32 = reinterpret_cast<float*>(ws + bp.off_q32);
  float* qx32 = reinterpret_cast<float*>(ws + bp.off_qx32);
  float* lsyn = reinterpret_cast<float*>(ws + bp.off_lsyn);
  float* z32 = reinterpret_cast<float*>(ws + bp.off_z32);
  float* lenc = reinterpret_cast<float*>(ws + bp.off_lenc);
  float* ltok = reinterpret_cast<float*>(ws + bp.off_ltok);
  float* dtok = reinterpret_cast<float*>(ws + bp.off_dtok);
  float* dz32 = reinterpret_cast<float*>(ws + bp.off_dz32);
  float* gam = reinterpret_cast<float*>(ws + bp.off_gam);
  float* dqx32 = reinterpret_cast<float*>(ws + bp.off_dqx32);
  float* dqxdec = reinterpret_cast<float*>(ws + bp.off_dqxdec);
  float* gsyn = reinterpret_cast<float*>(ws + bp.off_gsyn);
  float* qpad = reinterpret_cast<float*>(ws + bp.off_qpad);
  float* zpad = reinterpret_cast<float*>(ws + bp.off_zpad);
  float* dzpad = reinterpret_cast<float*>(ws + bp.off_dzpad);
  float* q0pad = reinterpret_cast<float*>(ws + bp.off_q0pad);
  float* dqxpad = reinterpret_cast<float*>(ws + bp.off_dqxpad);
  float* g32 = reinterpret_cast<float*>(ws + bp.off_g32);
  const size_t P = part_floats(bp, B, H, M, D, false);
  const size_t stride = pp_exchange_floats(bp, phase - 1, B, H, M, D, C);  // of the gathered buffers
  flare_status st = FLARE_OK;
  switch (phase) {
    case 0: {
      if (cudaMemsetAsync(ws + bp.fwd.off_err, 0, 8, s) != cudaSuccess) return FLARE_ERR_LAUNCH;
      // eq. 7 and 9: the projections, recomputed (tcgen05, as in the forward)
      Projected pr;
      if ((st = flarepp_project(bp.fwd, a.X, a.Wk, a.Wv, a.Wk_syn, a.Wv_syn, B, N, C, H, D, ws, s, nullptr, &pr)) !=
          FLARE_OK)
        return st;
      const CvtParams cv{static_cast<long>(H) * M * D, reinterpret_cast<const uint16_t*>(a.Q0), q32};
      if (launch_cvt(cv, s) != cudaSuccess) return FLARE_ERR_LAUNCH;
      // eq. 8 recomputed: the synthesis partials of this shard
      LatParams lf = lat_params(bp, ws, q32, 0, kt, B, H, N, M, D, a.lengths, sc, a.sh);
      lf.v = vt;
      lf.part_a = exch;
      return launch_lat(kLatForward, lf, s) == cudaSuccess ? FLARE_OK : FLARE_ERR_LAUNCH;
    }
    case 1: {
      if ((st = lat_merge(gathered, R, stride, static_cast<int>(BH), M, D, bp.S, qx32, lsyn, s)) != FLARE_OK)
        return st;
      // eq. 10 recomputed: the encode partials of this shard
      LatParams lf = lat_params(bp, ws, qx32, 1, kk, B, H, N, M, D, a.lengths, sc, a.sh);
      lf.v = vv;
      lf.part_a = exch;
      return launch_lat(kLatForward, lf, s) == cudaSuccess ? FLARE_OK : FLARE_ERR_LAUNCH;
    }
    case 2: {
      if ((st = lat_merge(gathered, R, stride, static_cast<int>(BH), M, D, bp.S, z32, lenc, s)) != FLARE_OK ||
          (st = pad(qx32, qpad, BH * M, D, c, s)) != FLARE_OK || (st = pad(z32, zpad, BH * M, D, 1.f, s)) != FLARE_OK)
        return st;
      // eq. 11: the decoder's per-token normalisers and delta_n
      TokParams tp = tok_params(B, H, N, M, D, 1, a.lengths, sc, a.sh);
      tp.qpad = qpad; tp.zpad = zpad;
      tp.k = kk; tp.dy = reinterpret_cast<const uint16_t*>(a.dY);
      tp.ltok = ltok; tp.dtok = dtok;
      if (launch_tok(kTokStats, tp, s) != cudaSuccess) return FLARE_ERR_LAUNCH;
      // decoder backward, reductions over this shard's tokens: dZ and dQ(X) partials
      LatParams ld = lat_params(bp, ws, qx32, 1, kk, B, H, N, M, D, a.lengths, sc, a.sh);
      ld.zrow = z32; ld.dy = tp.dy; ld.ltok = ltok; ld.dtok = dtok;
      ld.part_a = exch; ld.part_b = exch + P;
      return launch_lat(kLatDecoder, ld, s) == cudaSuccess ? FLARE_OK : FLARE_ERR_LAUNCH;
    }
    case 3: {
      // dZ and gamma; the decoder's part of dQ(X)
      if ((st = lat_sum(B, H, M, D, bp.S, 0, 1.f, gathered, nullptr, R, stride, nullptr, z32, gam, dz32, s)) !=
              FLARE_OK ||
          (st = lat_sum(B, H, M, D, bp.S, 0, sc, gathered + P, nullptr, R, stride, nullptr, nullptr, nullptr,
                        dqxdec, s)) != FLARE_OK ||
          (st = pad(dz32, dzpad, BH * M, D, 1.f, s)) != FLARE_OK)
        return st;
      // dK (both parts) and dV of this shard's tokens, into the gradient rows
      TokParams tp = tok_params(B, H, N, M, D, 1, a.lengths, sc, a.sh);
      tp.qpad = qpad; tp.zpad = zpad; tp.dzpad = dzpad; tp.lm = lenc; tp.gam = gam;
      tp.k = kk; tp.v = vv; tp.dy = reinterpret_cast<const uint16_t*>(a.dY);
      tp.ltok = ltok; tp.dtok = dtok;
      tp.g32 = g32; tp.g_ld = 4 * C; tp.g_col_k = 0; tp.g_col_v = C;
      if (launch_tok(kTokFull, tp, s) != cudaSuccess) return FLARE_ERR_LAUNCH;
      // encoder backward: its dQ(X) partials
      LatParams le = lat_params(bp, ws, qx32, 1, kk, B, H, N, M, D, a.lengths, sc, a.sh);
      le.zrow = dz32; le.lrow = lenc; le.grow = gam; le.v = vv;
      le.part_b = exch;
      return launch_lat(kLatEncoder, le, s) == cudaSuccess ? FLARE_OK : FLARE_ERR_LAUNCH;
    }
    case 4: {
      // dQ(X) = scale * (decoder + encoder parts); gamma of the synthesis
      if ((st = lat_sum(B, H, M, D, bp.S, 0, sc, gathered, nullptr, R, stride, dqxdec, qx32, gsyn, dqx32, s)) !=
              FLARE_OK ||
          (st = pad(q32, q0pad, static_cast<long>(H) * M, D, c, s)) != FLARE_OK ||
          (st = pad(dqx32, dqxpad, BH * M, D, 1.f, s)) != FLARE_OK)
        return st;
      // eq. 8 backward with dQ(X) as the upstream gradient: dK~, dV~ rows ...
      TokParams tp = tok_params(B, H, N, M, D, 0, a.lengths, sc, a.sh);
      tp.qpad = q0pad; tp.dzpad = dqxpad; tp.lm = lsyn; tp.gam = gsyn;
      tp.k = kt; tp.v = vt;
      tp.g32 = g32; tp.g_ld = 4 * C; tp.g_col_k = 2 * C; tp.g_col_v = 3 * C;
      if (launch_tok(kTokEncoder, tp, s) != cudaSuccess) return FLARE_ERR_LAUNCH;
      // ... and the partials of dQ0
      LatParams le = lat_params(bp, ws, q32, 0, kt, B, H, N, M, D, a.lengths, sc, a.sh);
      le.zrow = dqx32; le.lrow = lsyn; le.grow = gsyn; le.v = vt;
      le.part_b = exch;
      return launch_lat(kLatEncoder, le, s) == cudaSuccess ? FLARE_OK : FLARE_ERR_LAUNCH;
    }
    case 5: {
      // dQ0, summed over the batch and the shards
      if ((st = lat_sum(B, H, M, D, bp.S, 1, sc, gathered, nullptr, R, stride, nullptr, nullptr, nullptr, a.dQ0, s)) !=
          FLARE_OK)
        return st;
      // projections backward on this shard's rows: dX = G [Wk | Wv | Wk~ | Wv~]^T, partials of X^T G
      const long rows = static_cast<long>(B) * N;
      DxParams dx{};
      dx.R = static_cast<int>(rows); dx.C = C; dx.nw = 4;
      dx.g = g32;
      const flare_bf16* w4[4] = {a.Wk, a.Wv, a.Wk_syn, a.Wv_syn};
      for (int i = 0; i < 4; ++i) dx.w[i] = reinterpret_cast<const uint16_t*>(w4[i]);
      dx.dx = reinterpret_cast<uint16_t*>(a.dX);
      if (launch_dx(dx, s) != cudaSuccess) return FLARE_ERR_LAUNCH;
      const DwParams dw{static_cast<int>(rows), C, 4 * C, bp.dw_splits, reinterpret_cast<const uint16_t*>(a.X), g32,
                        exch};
      return launch_dw(dw, s) == cudaSuccess ? FLARE_OK : FLARE_ERR_LAUNCH;
    }
    case 6: {
      // dW: the partials of every shard's rows (rank-major, so the splits of all
      // shards form one ascending sequence)
      DwReduceParams dr{};
      dr.C = C; dr.J = 4 * C; dr.n_splits = R * bp.dw_splits; dr.shared = shared ? 1 : 0;
      dr.part = gathered;
      dr.dw[0] = a.dWk; dr.dw[1] = a.dWv; dr.dw[2] = a.dWk_syn; dr.dw[3] = a.dWv_syn;
      return launch_dw_reduce(dr, s) == cudaSuccess ? FLARE_OK : FLARE_ERR_LAUNCH;
    }
    default:
      return FLARE_ERR_SHAPE;
  }
}

flare_status check_bwd_sizes(int B, int H, int N, int M, int D) {
  flare_status st = check_common(B, H, N, M, D);
  if (st != FLARE_OK) return st;
  return static_cast<long>(B) * H > 65535 ? FLARE_ERR_UNSUPPORTED : FLARE_OK;
}

// Checks shared by the FLARE++ backward entry points.
flare_status check_pp_bwd(const PpArgs& a, const void* workspace) {
  flare_status st = check_flarepp(a.X, a.Wk, a.Wv, a.Wk_syn, a.Wv_syn, a.Q0, a.dY, a.B, a.N, a.C, a.H, a.M, a.D,
                                  a.lengths, workspace, nullptr, nullptr);
  if (st != FLARE_OK) return st;
  const bool shared = a.Wk_syn == a.Wk && a.Wv_syn == a.Wv;
  if (!a.dX || !a.dWk || !a.dWv || !a.dQ0 || (!shared && (!a.dWk_syn || !a.dWv_syn))) return FLARE_ERR_NULL;
  if ((st = check_bwd_sizes(a.B, a.H, a.N, a.M, a.D)) != FLARE_OK) return st;
  if (static_cast<long>(a.B) * a.N > 65535L * kBwdDwRows) return FLARE_ERR_UNSUPPORTED;
  if (!aligned16(a.dX) || !aligned16(a.dWk) || !aligned16(a.dWv) || !aligned16(a.dWk_syn) || !aligned16(a.dWv_syn) ||
      !aligned16(a.dQ0))
    return FLARE_ERR_ALIGN;
  return FLARE_OK;
}

}  // namespace
}  // namespace flare

extern "C" {

flare_status flare_mixer_bwd(const flare_bf16* K, const flare_bf16* V, const flare_bf16* Q, const flare_bf16* dY,
                             flare_bf16* dK, flare_bf16* dV, float* dQ, int B, int H, int N, int M, int D,
                             const int32_t* lengths, float scale, void* workspace, size_t workspace_bytes,
                             void* stream) {
  if (!K || !V || !Q || !dY || !dK || !dV || !dQ || !workspace) return FLARE_ERR_NULL;
  flare_status st = check_bwd_sizes(B, H, N, M, D);
  if (st != FLARE_OK) return st;
  if (!aligned16(K) || !aligned16(V) || !aligned16(Q) || !aligned16(dY) || !aligned16(dK) || !aligned16(dV) ||
      !aligned16(dQ) || !aligned16(lengths) || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return FLARE_ERR_ALIGN;
  const BwdPlan bp = make_bwd_plan(false, B, H, N, M, D, 0);
  if (workspace_bytes < bp.total) return FLARE_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  if (cudaMemsetAsync(ws + bp.fwd.off_err, 0, 8, s) != cudaSuccess) return FLARE_ERR_LAUNCH;
  float* q32 = reinterpret_cast<float*>(ws + bp.off_q32);
  const CvtParams cv{static_cast<long>(H) * M * D, reinterpret_cast<const uint16_t*>(Q), q32};
  if (launch_cvt(cv, s) != cudaSuccess) return FLARE_ERR_LAUNCH;
  return flare_bwd_run(bp, ws, q32, K, V, dY, reinterpret_cast<uint16_t*>(dK), reinterpret_cast<uint16_t*>(dV), dQ, B,
                       H, N, M, D, lengths, resolve_scale(scale, D), s);
}

flare_status flarepp_mixer_bwd(const flare_bf16* X, const flare_bf16* Wk, const flare_bf16* Wv,
                               const flare_bf16* Wk_syn, const flare_bf16* Wv_syn, const flare_bf16* Q0,
                               const flare_bf16* dY, flare_bf16* dX, float* dWk, float* dWv, float* dWk_syn,
                               float* dWv_syn, float* dQ0, int B, int N, int C, int H, int M, int D,
                               const int32_t* lengths, float scale, void* workspace, size_t workspace_bytes,
                               void* stream) {
  const PpArgs a{X, Wk, Wv, Wk_syn, Wv_syn, Q0, dY, dX, dWk, dWv, dWk_syn, dWv_syn, dQ0,
                 B, N, C, H, M, D, lengths, resolve_scale(scale, D), Shard{0, N, 1}};
  flare_status st = check_pp_bwd(a, workspace);
  if (st != FLARE_OK) return st;
  const BwdPlan bp = make_bwd_plan(true, B, H, N, M, D, C);
  if (workspace_bytes < bp.total) return FLARE_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  // one shard: the exchanges stay in the workspace (stream order makes every
  // reuse safe: a buffer is read by the next phase's first launches before
  // that phase writes its own exchange)
  float* ex[kPpPhases - 1] = {reinterpret_cast<float*>(ws + bp.off_fpart), reinterpret_cast<float*>(ws + bp.off_fpart),
                              reinterpret_cast<float*>(ws + bp.off_pa),    reinterpret_cast<float*>(ws + bp.off_pc),
                              reinterpret_cast<float*>(ws + bp.off_pc),    reinterpret_cast<float*>(ws + bp.off_dwpart)};
  for (int ph = 0; ph < kPpPhases; ++ph) {
    st = pp_phase(ph, bp, ws, a, ph > 0 ? ex[ph - 1] : nullptr, ph < kPpPhases - 1 ? ex[ph] : nullptr, s);
    if (st != FLARE_OK) return st;
  }
  return FLARE_OK;
}

size_t flarepp_cp_bwd_exchange_bytes(int phase, int B, int N, int C, int H, int M, int D) {
  if (phase < 0 || phase >= kPpPhases - 1) return 0;
  if (check_bwd_sizes(B, H, N, M, D) != FLARE_OK || C != H * D || C % 64 != 0 || C > 256) return 0;
  return pp_exchange_floats(make_bwd_plan(true, B, H, N, M, D, C), phase, B, H, M, D, C) * sizeof(float);
}

flare_status flarepp_cp_bwd_phase(int phase, const flare_bf16* X, const flare_bf16* Wk, const flare_bf16* Wv,
                                  const flare_bf16* Wk_syn, const flare_bf16* Wv_syn, const flare_bf16* Q0,
                                  const flare_bf16* dY, const float* gathered, float* exchange, flare_bf16* dX,
                                  float* dWk, float* dWv, float* dWk_syn, float* dWv_syn, float* dQ0, int B, int N,
                                  int C, int H, int M, int D, const int32_t* lengths, int rank, int world,
                                  float scale, void* workspace, size_t workspace_bytes, void* stream) {
  if (phase < 0 || phase >= kPpPhases) return FLARE_ERR_SHAPE;
  if (world < 1 || rank < 0 || rank >= world) return FLARE_ERR_SHAPE;
  if (static_cast<long>(N) * world >= (1L << 31)) return FLARE_ERR_UNSUPPORTED;
  if ((phase > 0 && !gathered) || (phase < kPpPhases - 1 && !exchange)) return FLARE_ERR_NULL;
  if (!aligned16(gathered) || !aligned16(exchange)) return FLARE_ERR_ALIGN;
  const PpArgs a{X, Wk, Wv, Wk_syn, Wv_syn, Q0, dY, dX, dWk, dWv, dWk_syn, dWv_syn, dQ0,
                 B, N, C, H, M, D, lengths, resolve_scale(scale, D), Shard{rank * N, world * N, world}};
  flare_status st = check_pp_bwd(a, workspace);
  if (st != FLARE_OK) return st;
  const BwdPlan bp = make_bwd_plan(true, B, H, N, M, D, C);
  if (workspace_bytes < bp.total) return FLARE_ERR_WORKSPACE;
  return pp_phase(phase, bp, static_cast<uint8_t*>(workspace), a, gathered, exchange,
                  static_cast<cudaStream_t>(stream));
}

}  // extern "C"
