// Host entry points of the C ABI declared in include/flare.h, forward side:
// argument validation (before anything is enqueued), workspace layout, TMA
// tensor maps and the launch sequences of the FLARE / FLARE++ forward and of
// its context-parallel phases.  The backward's entry points are in
// api_bwd.cu; host_internal.h declares what the two share.
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "bwd_internal.h"
#include "flare.h"
#include "flare_internal.h"
#include "host_internal.h"

namespace flare {

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

// 2-D fp32 tensor map: dims (d0 innermost, d1), dense, box (b0, b1), no swizzle.
bool map2d_f32(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint32_t b0, uint32_t b1) {
  EncodeTiledFn fn = tensor_map_encoder();
  if (!fn) return false;
  const cuuint64_t dims[2] = {d0, d1};
  const cuuint64_t strides[1] = {d0 * 4};
  const cuuint32_t box[2] = {b0, b1};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}


// Number of token splits of the encoder.  Cost model: the CTAs run in
// waves of `slots` (CTAs resident on the whole GPU); a wave lasts as long as
// one split (its tiles plus a fixed set-up cost worth setup_tiles tiles).
// Depends on the sizes only, so a given problem always uses the same split
// count (and gives the same bits).
int choose_splits(long units, long ntiles, long slots, long setup_tiles) {
  const long smax = std::max(1L, std::min(ntiles, 1024L));
  int best = 1;
  long best_cost = -1;
  for (long s = 1; s <= smax; ++s) {
    const long tps = cdiv(ntiles, s);
    if (s > 1 && cdiv(ntiles, tps) < s) continue;  // same tiling as a smaller s
    const long cost = cdiv(units * s, slots) * (tps + setup_tiles);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = static_cast<int>(s);
    }
  }
  return best;
}


Plan make_plan(int variant, long B, long H, long N, long M, long D) {
  Plan p;
  const long BH = B * H;
  const long ntiles = cdiv(N, enc_tile(static_cast<int>(D)));
  p.LB = static_cast<int>(cdiv(M, kLatBlock));
  // an encoder CTA's set-up (TMEM allocation, barriers, the first tiles of
  // its pipeline) costs about as much as 384 tokens of work
  p.S = choose_splits(BH * p.LB, ntiles, static_cast<long>(kNumSM) * enc_ctas_per_sm(static_cast<int>(D)),
                      cdiv(384, enc_tile(static_cast<int>(D))));
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

// Records stage event i (a cudaEvent_t passed as void*) when profiling is on.
bool record(void* const* ev, int i, cudaStream_t s) {
  if (ev == nullptr || ev[i] == nullptr) return true;
  return cudaEventRecord(static_cast<cudaEvent_t>(ev[i]), s) == cudaSuccess;
}


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
                                 void* const* ev, int ev0, bool pdl) {
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
  if (launch_encode(tq, tk, tv, ep, st, pdl) != cudaSuccess || !record(ev, ev0, st)) return FLARE_ERR_LAUNCH;
  return FLARE_OK;
}

// Merge of the partials of R shards ([R][B*H][S][M][D+2], rank-major) into
// out32/out16 ([B*H][M][D]).  With R == 1, q/k/v serve the exact
// recomputation of rows whose sums underflowed.
// exact: every shard's exact partials of the rows that need them
// ([R][B*H*M][D+2], context parallelism), or nullptr.
MergeParams merge_params(const Plan& pl, uint8_t* ws, const float* part, int R, const void* q, int q_per_batch,
                         const void* k, const void* v, float* out32, uint16_t* out16, int B, int H, int N, int M,
                         int D, const int32_t* lengths, float scale, bool allow_exact, const float* exact) {
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
  mp.fix = exact;
  mp.fix_rank_stride = static_cast<size_t>(B) * H * M * (D + 2);
  return mp;
}

flare_status run_merge(const Plan& pl, uint8_t* ws, const float* part, int R, const void* q, int q_per_batch,
                       const void* k, const void* v, float* out32, uint16_t* out16, int B, int H, int N, int M,
                       int D, const int32_t* lengths, float scale, cudaStream_t st, void* const* ev, int ev_i,
                       bool pdl, bool allow_exact = true, const float* exact = nullptr, float* lse_out = nullptr) {
  MergeParams mp =
      merge_params(pl, ws, part, R, q, q_per_batch, k, v, out32, out16, B, H, N, M, D, lengths, scale, allow_exact, exact);
  mp.lse_out = lse_out;
  if (launch_merge(mp, st, pdl) != cudaSuccess || !record(ev, ev_i, st)) return FLARE_ERR_LAUNCH;
  return FLARE_OK;
}

// Context parallelism: this shard's exact partials (out, [B*H*M][D+2]) of
// the rows whose merge of the gathered partials `part` needs them.
flare_status run_cp_exact(const Plan& pl, uint8_t* ws, const float* part, int R, int rank, const void* q,
                          int q_per_batch, const void* k, const void* v, int B, int H, int N, int M, int D,
                          const int32_t* lengths, float scale, cudaStream_t st, float* out) {
  const MergeParams mp = merge_params(pl, ws, part, R, q, q_per_batch, k, v, nullptr, nullptr, B, H, N, M, D,
                                      lengths, scale, false, nullptr);
  return launch_cp_exact(mp, rank, out, st) == cudaSuccess ? FLARE_OK : FLARE_ERR_LAUNCH;
}

// Encoder pass + merge on one GPU (the whole sequence).
flare_status run_encode(const Plan& pl, uint8_t* ws, const void* q, int q_per_batch, const void* k, const void* v,
                        const float* knorm, float* out32, uint16_t* out16, int B, int H, int N, int M, int D,
                        const int32_t* lengths, float scale, cudaStream_t st, void* const* ev, int ev0, bool pdl,
                        float* lse_out = nullptr) {
  float* part = reinterpret_cast<float*>(ws + pl.off_part);
  flare_status r = run_encode_partials(pl, ws, q, q_per_batch, k, v, knorm, part, B, H, N, M, D, lengths, 0, N,
                                       scale, st, ev, ev0, pdl);
  if (r != FLARE_OK) return r;
  return run_merge(pl, ws, part, 1, q, q_per_batch, k, v, out32, out16, B, H, N, M, D, lengths, scale, st, ev,
                   ev0 + 1, pdl, true, nullptr, lse_out);
}

flare_status run_decode(const Plan& pl, uint8_t* ws, const void* q, int q_per_batch, const uint16_t* z16,
                        const void* k, void* y, int y_token_major, int B, int H, int N, int M, int D,
                        const int32_t* lengths, float scale, cudaStream_t st, bool pdl, int tok_offset = 0,
                        int n_global = -1, float* y_f32 = nullptr, int z_f16 = 0, const float* z32 = nullptr,
                        float* ltok_out = nullptr) {
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
  dp.y_f32 = y_f32;
  dp.z_f16 = z_f16;
  dp.z32 = z32;
  dp.ltok_out = ltok_out;
  dp.tok_offset = tok_offset;
  dp.n_global = n_global < 0 ? N : n_global;
  dp.err = reinterpret_cast<uint32_t*>(ws + pl.off_err);
  dp.fb_count = reinterpret_cast<uint32_t*>(ws + pl.off_err) + 1;
  dp.fb_list = reinterpret_cast<uint64_t*>(ws + pl.off_fb);
  dp.timeout_ns = wait_timeout_ns();
  if (launch_decode(tq, tz, tk, dp, st, pdl) != cudaSuccess) return FLARE_ERR_LAUNCH;
  return FLARE_OK;
}

}  // namespace flare

namespace flare {

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
    case FLARE_ERR_NO_FORWARD:
      return "FLARE_ERR_NO_FORWARD: a training backward found no training forward's state in its workspace";
  }
  return "unknown flare_status";
}

}  // extern "C"

namespace flare {

// The FLARE forward (eq. 5-6) after nothing but the caller's arguments:
// A training forward's decoder (FwdStats with zf16, D = 16) takes Z in fp16:
// convert the merged fp32 Z first.
flare_status train_decode_inputs(const FwdStats* stats, const float* z32, int B, int H, int M, int D, cudaStream_t s) {
  if (stats == nullptr || stats->zf16 == nullptr) return FLARE_OK;
  if (D != 16) return FLARE_ERR_UNSUPPORTED;
  const ToF16Params tp{static_cast<long>(B) * H * M * D, z32, stats->zf16};
  return launch_to_f16(tp, s) == cudaSuccess ? FLARE_OK : FLARE_ERR_LAUNCH;
}

// checks, then key norms | encode | merge | decode on `stream`.
flare_status flare_fwd(const flare_bf16* K, const flare_bf16* V, const flare_bf16* Q, flare_bf16* Y, int B, int H,
                       int N, int M, int D, const int32_t* lengths, float scale, void* workspace,
                       size_t workspace_bytes, void* stream, float* Z_out, float* Y_f32_out,
                       void* const* stage_events, const FwdStats* stats) {
  // Y may be null only for a training forward run inside a backward call,
  // which needs the kept state and not Y
  if (!K || !V || !Q || (!Y && !stats) || !workspace) return FLARE_ERR_NULL;
  flare_status st = check_common(B, H, N, M, D);
  if (st != FLARE_OK) return st;
  if (!aligned16(K) || !aligned16(V) || !aligned16(Q) || !aligned16(Y) || !aligned16(lengths) || !aligned16(Z_out) ||
      !aligned16(Y_f32_out) || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return FLARE_ERR_ALIGN;
  const Plan pl = make_plan(FLARE_VARIANT_FLARE, B, H, N, M, D);
  if (workspace_bytes < pl.total) return FLARE_ERR_WORKSPACE;
  const float sc = resolve_scale(scale, D);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  if (cudaMemsetAsync(ws + pl.off_err, 0, kErrClearBytes, s) != cudaSuccess) return FLARE_ERR_LAUNCH;
  if (!record(stage_events, 0, s)) return FLARE_ERR_LAUNCH;
  KnormParams kp{B * H, N, D, pl.G32, reinterpret_cast<const uint16_t*>(K), reinterpret_cast<float*>(ws + pl.off_kn)};
  if (launch_knorm(kp, s) != cudaSuccess || !record(stage_events, 1, s)) return FLARE_ERR_LAUNCH;
  float* z32 = Z_out ? Z_out : reinterpret_cast<float*>(ws + pl.off_z32);
  uint16_t* z16 = reinterpret_cast<uint16_t*>(ws + pl.off_z16);
  // kernels after the first start early (programmatic launch) unless stage
  // events sit between them
  const bool pdl = stage_events == nullptr;
  st = run_encode(pl, ws, Q, 0, K, V, kp.knorm, z32, z16, B, H, N, M, D, lengths, sc, s, stage_events, 2, pdl,
                  stats ? stats->lenc : nullptr);
  if (st != FLARE_OK) return st;
  st = train_decode_inputs(stats, z32, B, H, M, D, s);
  if (st != FLARE_OK) return st;
  const bool f16 = stats != nullptr && stats->zf16 != nullptr;
  st = run_decode(pl, ws, Q, 0, f16 ? stats->zf16 : z16, K, Y, 0, B, H, N, M, D, lengths, sc, s, pdl, 0, -1,
                  f16 ? stats->y32 : Y_f32_out, f16 ? 1 : 0, f16 ? z32 : nullptr, f16 ? stats->ltok : nullptr);
  if (st != FLARE_OK) return st;
  return record(stage_events, 4, s) ? FLARE_OK : FLARE_ERR_LAUNCH;
}

}  // namespace flare

extern "C" {

flare_status flare_mixer_fwd_profiled(const flare_bf16* K, const flare_bf16* V, const flare_bf16* Q, flare_bf16* Y,
                                      int B, int H, int N, int M, int D, const int32_t* lengths, float scale,
                                      void* workspace, size_t workspace_bytes, void* stream, float* Z_out,
                                      void* const* stage_events) {
  return flare_fwd(K, V, Q, Y, B, H, N, M, D, lengths, scale, workspace, workspace_bytes, stream, Z_out, nullptr,
                   stage_events, nullptr);
}

flare_status flare_mixer_fwd_inspect(const flare_bf16* K, const flare_bf16* V, const flare_bf16* Q, flare_bf16* Y,
                                     int B, int H, int N, int M, int D, const int32_t* lengths, float scale,
                                     void* workspace, size_t workspace_bytes, void* stream, float* Z_out,
                                     float* Y_f32_out) {
  if (!Y_f32_out) return FLARE_ERR_NULL;
  return flare_fwd(K, V, Q, Y, B, H, N, M, D, lengths, scale, workspace, workspace_bytes, stream, Z_out, Y_f32_out,
                   nullptr, nullptr);
}

flare_status flare_mixer_fwd(const flare_bf16* K, const flare_bf16* V, const flare_bf16* Q, flare_bf16* Y, int B,
                             int H, int N, int M, int D, const int32_t* lengths, float scale, void* workspace,
                             size_t workspace_bytes, void* stream, float* Z_out) {
  return flare_mixer_fwd_profiled(K, V, Q, Y, B, H, N, M, D, lengths, scale, workspace, workspace_bytes, stream,
                                  Z_out, nullptr);
}

}  // extern "C"

namespace flare {

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
                         int H, int D, cudaStream_t s, bool pdl) {
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
  return launch_project(tx, tw, pp, s, pdl) == cudaSuccess ? FLARE_OK : FLARE_ERR_LAUNCH;
}


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
  flare_status st = run_project(pl, ws, tx, tw, shared ? 2 : 4, 0, outs, norms, B, N, C, H, D, s, false);
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
                         void* const* stage_events, float* Y_f32_out, const FwdStats* stats) {
  if (cudaMemsetAsync(ws + pl.off_err, 0, kErrClearBytes, s) != cudaSuccess) return FLARE_ERR_LAUNCH;
  Projected pr;
  flare_status st = flarepp_project(pl, X, Wk, Wv, Wk_syn, Wv_syn, B, N, C, H, D, ws, s, stage_events, &pr);
  if (st != FLARE_OK) return st;
  uint16_t *kt = pr.kt, *vt = pr.vt, *kk = pr.kk, *vv = pr.vv;
  float *kn_syn = pr.kn_syn, *kn = pr.kn;

  // kernels after the first start early (programmatic launch) unless stage
  // events sit between them
  const bool pdl = stage_events == nullptr;
  // eq. 8: query synthesis with the learned seeds
  float* qx32 = Qx_out ? Qx_out : reinterpret_cast<float*>(ws + pl.off_qx32);
  uint16_t* qx16 = reinterpret_cast<uint16_t*>(ws + pl.off_qx16);
  st = run_encode(pl, ws, Q0, 0, kt, vt, kn_syn, qx32, qx16, B, H, N, M, D, lengths, sc, s, stage_events, 2, pdl,
                  stats ? stats->lsyn : nullptr);
  if (st != FLARE_OK) return st;
  // eq. 10: encode with the synthesised queries
  float* z32 = Z_out ? Z_out : reinterpret_cast<float*>(ws + pl.off_z32);
  uint16_t* z16 = reinterpret_cast<uint16_t*>(ws + pl.off_z16);
  st = run_encode(pl, ws, qx16, 1, kk, vv, kn, z32, z16, B, H, N, M, D, lengths, sc, s, stage_events, 4, pdl,
                  stats ? stats->lenc : nullptr);
  if (st != FLARE_OK) return st;
  // eq. 11: decode
  st = train_decode_inputs(stats, z32, B, H, M, D, s);
  if (st != FLARE_OK) return st;
  const bool f16 = stats != nullptr && stats->zf16 != nullptr;
  st = run_decode(pl, ws, qx16, 1, f16 ? stats->zf16 : z16, kk, Y, y_token_major, B, H, N, M, D, lengths, sc, s, pdl,
                  0, -1, f16 ? stats->y32 : Y_f32_out, f16 ? 1 : 0, f16 ? z32 : nullptr,
                  f16 ? stats->ltok : nullptr);
  if (st != FLARE_OK) return st;
  return record(stage_events, 6, s) ? FLARE_OK : FLARE_ERR_LAUNCH;
}

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
                     stage_events, nullptr, nullptr);
}

flare_status flarepp_mixer_fwd_inspect(const flare_bf16* X, const flare_bf16* Wk, const flare_bf16* Wv,
                                       const flare_bf16* Wk_syn, const flare_bf16* Wv_syn, const flare_bf16* Q0,
                                       flare_bf16* Y, int B, int N, int C, int H, int M, int D,
                                       const int32_t* lengths, float scale, void* workspace, size_t workspace_bytes,
                                       void* stream, float* Qx_out, float* Z_out, float* Y_f32_out) {
  if (!Y_f32_out) return FLARE_ERR_NULL;
  flare_status st = check_flarepp(X, Wk, Wv, Wk_syn, Wv_syn, Q0, Y, B, N, C, H, M, D, lengths, workspace, Qx_out,
                                  Z_out);
  if (st != FLARE_OK) return st;
  if (!aligned16(Y_f32_out)) return FLARE_ERR_ALIGN;
  const Plan pl = make_plan(FLARE_VARIANT_FLAREPP, B, H, N, M, D);
  if (workspace_bytes < pl.total) return FLARE_ERR_WORKSPACE;
  return flarepp_run(pl, X, Wk, Wv, Wk_syn, Wv_syn, Q0, Y, 0, B, N, C, H, M, D, lengths, resolve_scale(scale, D),
                     static_cast<uint8_t*>(workspace), static_cast<cudaStream_t>(stream), Qx_out, Z_out, nullptr,
                     Y_f32_out, nullptr);
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
                   ws, s, nullptr, nullptr, nullptr, nullptr, nullptr);
  if (st != FLARE_OK) return st;
  // Out = concat_h(Y_h) W_O: the same tcgen05 projection with one weight and
  // token-major output rows
  CUtensorMap ty, two[4];
  if (!map3d(&ty, ycat, C, N, B, 64, kProjTile, CU_TENSOR_MAP_SWIZZLE_128B)) return FLARE_ERR_LAUNCH;
  for (int i = 0; i < 4; ++i)
    if (!map2d(&two[i], Wo, C, C, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B)) return FLARE_ERR_LAUNCH;
  uint16_t* const outs[4] = {Out, nullptr, nullptr, nullptr};
  float* const norms[4] = {nullptr, nullptr, nullptr, nullptr};
  return run_project(pl, ws, ty, two, 1, 1, outs, norms, B, N, C, H, D, s, true);
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

size_t flare_cp_exact_bytes(int B, int H, int M, int D) {
  if (check_common(B, H, 1, M, D) != FLARE_OK) return 0;
  return static_cast<size_t>(B) * H * M * (D + 2) * sizeof(float);
}

}  // extern "C"

namespace flare {

flare_status check_cp(int N, int rank, int world, const void* part) {
  if (!part) return FLARE_ERR_NULL;
  if (world < 1 || rank < 0 || rank >= world) return FLARE_ERR_SHAPE;
  if (static_cast<long>(N) * world >= (1L << 31)) return FLARE_ERR_UNSUPPORTED;
  if (!aligned16(part)) return FLARE_ERR_ALIGN;
  return FLARE_OK;
}

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
  if (cudaMemsetAsync(ws + pl.off_err, 0, kErrClearBytes, s) != cudaSuccess) return FLARE_ERR_LAUNCH;
  Projected pr;
  if ((st = flarepp_project(pl, X, Wk, Wv, Wk_syn, Wv_syn, B, N, C, H, D, ws, s, nullptr, &pr)) != FLARE_OK)
    return st;
  // eq. 8 on the local shard: the synthesis partials
  return run_encode_partials(pl, ws, Q0, 0, pr.kt, pr.vt, pr.kn_syn, partials, B, H, N, M, D, lengths, rank * N,
                             world * N, resolve_scale(scale, D), s, nullptr, 0, true);
}

flare_status flarepp_cp_middle(const float* partials_all, const float* exact_all, int B, int N, int C, int H, int M,
                               int D, const int32_t* lengths, int rank, int world, float scale, void* workspace,
                               size_t workspace_bytes, void* stream, float* partials, float* Qx_out) {
  if (!partials_all || !workspace) return FLARE_ERR_NULL;
  flare_status st = check_common(B, H, N, M, D);
  if (st != FLARE_OK) return st;
  if (C != H * D || C % 64 != 0 || C > 256) return C != H * D ? FLARE_ERR_SHAPE : FLARE_ERR_UNSUPPORTED;
  if ((st = check_cp(N, rank, world, partials)) != FLARE_OK) return st;
  if (!aligned16(partials_all) || !aligned16(exact_all) || !aligned16(lengths) || !aligned16(Qx_out))
    return FLARE_ERR_ALIGN;
  const Plan pl = make_plan(FLARE_VARIANT_FLAREPP, B, H, N, M, D);
  if (workspace_bytes < pl.total) return FLARE_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const float sc = resolve_scale(scale, D);
  float* qx32 = Qx_out ? Qx_out : reinterpret_cast<float*>(ws + pl.off_qx32);
  uint16_t* qx16 = reinterpret_cast<uint16_t*>(ws + pl.off_qx16);
  // Q(X): every rank merges the same partials in the same order
  st = run_merge(pl, ws, partials_all, world, nullptr, 0, nullptr, nullptr, qx32, qx16, B, H, N, M, D, lengths, sc, s,
                 nullptr, 0, false, false, exact_all);
  if (st != FLARE_OK) return st;
  // eq. 10 on the local shard: the encode partials
  return run_encode_partials(pl, ws, qx16, 1, ws + pl.off_kp, ws + pl.off_vp, reinterpret_cast<float*>(ws + pl.off_kn),
                             partials, B, H, N, M, D, lengths, rank * N, world * N, sc, s, nullptr, 0, true);
}

flare_status flarepp_cp_end(const float* partials_all, const float* exact_all, flare_bf16* Y, int B, int N, int C,
                            int H, int M, int D, const int32_t* lengths, int rank, int world, float scale,
                            void* workspace, size_t workspace_bytes, void* stream, float* Z_out) {
  if (!partials_all || !Y || !workspace) return FLARE_ERR_NULL;
  flare_status st = check_common(B, H, N, M, D);
  if (st != FLARE_OK) return st;
  if (C != H * D || C % 64 != 0 || C > 256) return C != H * D ? FLARE_ERR_SHAPE : FLARE_ERR_UNSUPPORTED;
  if ((st = check_cp(N, rank, world, partials_all)) != FLARE_OK) return st;
  if (!aligned16(Y) || !aligned16(exact_all) || !aligned16(lengths) || !aligned16(Z_out)) return FLARE_ERR_ALIGN;
  const Plan pl = make_plan(FLARE_VARIANT_FLAREPP, B, H, N, M, D);
  if (workspace_bytes < pl.total) return FLARE_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const float sc = resolve_scale(scale, D);
  float* z32 = Z_out ? Z_out : reinterpret_cast<float*>(ws + pl.off_z32);
  uint16_t* z16 = reinterpret_cast<uint16_t*>(ws + pl.off_z16);
  st = run_merge(pl, ws, partials_all, world, nullptr, 0, nullptr, nullptr, z32, z16, B, H, N, M, D, lengths, sc, s,
                 nullptr, 0, false, false, exact_all);
  if (st != FLARE_OK) return st;
  // eq. 11 on the local shard
  return run_decode(pl, ws, ws + pl.off_qx16, 1, z16, ws + pl.off_kp, Y, 0, B, H, N, M, D, lengths, sc, s, true,
                    rank * N, world * N);
}

flare_status flarepp_cp_exact(int pass, const float* partials_all, const flare_bf16* Wk, const flare_bf16* Wv,
                              const flare_bf16* Wk_syn, const flare_bf16* Wv_syn, const flare_bf16* Q0, int B, int N,
                              int C, int H, int M, int D, const int32_t* lengths, int rank, int world, float scale,
                              void* workspace, size_t workspace_bytes, void* stream, float* exact_out) {
  if (pass != 0 && pass != 1) return FLARE_ERR_SHAPE;
  if (!partials_all || !exact_out || !workspace || !Wk || !Wv || !Wk_syn || !Wv_syn || !Q0) return FLARE_ERR_NULL;
  flare_status st = check_common(B, H, N, M, D);
  if (st != FLARE_OK) return st;
  if (C != H * D || C % 64 != 0 || C > 256) return C != H * D ? FLARE_ERR_SHAPE : FLARE_ERR_UNSUPPORTED;
  if ((st = check_cp(N, rank, world, partials_all)) != FLARE_OK) return st;
  if (!aligned16(exact_out) || !aligned16(lengths) || !aligned16(Q0) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return FLARE_ERR_ALIGN;
  const Plan pl = make_plan(FLARE_VARIANT_FLAREPP, B, H, N, M, D);
  if (workspace_bytes < pl.total) return FLARE_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const bool shared = Wk_syn == Wk && Wv_syn == Wv;  // the synthesis used K and V (as in flarepp_cp_begin)
  if (pass == 0)
    return run_cp_exact(pl, ws, partials_all, world, rank, Q0, 0, ws + (shared ? pl.off_kp : pl.off_kt),
                        ws + (shared ? pl.off_vp : pl.off_vt), B, H, N, M, D, lengths, resolve_scale(scale, D),
                        static_cast<cudaStream_t>(stream), exact_out);
  return run_cp_exact(pl, ws, partials_all, world, rank, ws + pl.off_qx16, 1, ws + pl.off_kp, ws + pl.off_vp, B, H, N,
                      M, D, lengths, resolve_scale(scale, D), static_cast<cudaStream_t>(stream), exact_out);
}

flare_status flare_cp_exact(const float* partials_all, const flare_bf16* K, const flare_bf16* V, const flare_bf16* Q,
                            int B, int H, int N, int M, int D, const int32_t* lengths, int rank, int world,
                            float scale, void* workspace, size_t workspace_bytes, void* stream, float* exact_out) {
  if (!partials_all || !exact_out || !workspace || !K || !V || !Q) return FLARE_ERR_NULL;
  flare_status st = check_common(B, H, N, M, D);
  if (st != FLARE_OK) return st;
  if ((st = check_cp(N, rank, world, partials_all)) != FLARE_OK) return st;
  if (!aligned16(exact_out) || !aligned16(K) || !aligned16(V) || !aligned16(Q) || !aligned16(lengths) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return FLARE_ERR_ALIGN;
  const Plan pl = make_plan(FLARE_VARIANT_FLARE, B, H, N, M, D);
  if (workspace_bytes < pl.total) return FLARE_ERR_WORKSPACE;
  return run_cp_exact(pl, static_cast<uint8_t*>(workspace), partials_all, world, rank, Q, 0, K, V, B, H, N, M, D,
                      lengths, resolve_scale(scale, D), static_cast<cudaStream_t>(stream), exact_out);
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
  if (cudaMemsetAsync(ws + pl.off_err, 0, kErrClearBytes, s) != cudaSuccess) return FLARE_ERR_LAUNCH;
  KnormParams kp{B * H, N, D, pl.G32, reinterpret_cast<const uint16_t*>(K), reinterpret_cast<float*>(ws + pl.off_kn)};
  if (launch_knorm(kp, s) != cudaSuccess) return FLARE_ERR_LAUNCH;
  return run_encode_partials(pl, ws, Q, 0, K, V, kp.knorm, partials, B, H, N, M, D, lengths, rank * N, world * N,
                             resolve_scale(scale, D), s, nullptr, 0, true);
}

flare_status flare_cp_end(const float* partials_all, const float* exact_all, const flare_bf16* K, const flare_bf16* Q,
                          flare_bf16* Y, int B, int H, int N, int M, int D, const int32_t* lengths, int rank, int world,
                          float scale, void* workspace, size_t workspace_bytes, void* stream, float* Z_out) {
  if (!partials_all || !K || !Q || !Y || !workspace) return FLARE_ERR_NULL;
  flare_status st = check_common(B, H, N, M, D);
  if (st != FLARE_OK) return st;
  if ((st = check_cp(N, rank, world, partials_all)) != FLARE_OK) return st;
  if (!aligned16(K) || !aligned16(Q) || !aligned16(Y) || !aligned16(exact_all) || !aligned16(lengths) ||
      !aligned16(Z_out))
    return FLARE_ERR_ALIGN;
  const Plan pl = make_plan(FLARE_VARIANT_FLARE, B, H, N, M, D);
  if (workspace_bytes < pl.total) return FLARE_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const float sc = resolve_scale(scale, D);
  float* z32 = Z_out ? Z_out : reinterpret_cast<float*>(ws + pl.off_z32);
  uint16_t* z16 = reinterpret_cast<uint16_t*>(ws + pl.off_z16);
  st = run_merge(pl, ws, partials_all, world, nullptr, 0, nullptr, nullptr, z32, z16, B, H, N, M, D, lengths, sc, s,
                 nullptr, 0, false, false, exact_all);
  if (st != FLARE_OK) return st;
  return run_decode(pl, ws, Q, 0, z16, K, Y, 0, B, H, N, M, D, lengths, sc, s, true, rank * N, world * N);
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
  if (word & FLARE_DEV_NO_STATE) return FLARE_ERR_NO_FORWARD;
  return FLARE_OK;
}

flare_status flare_static_last_device_status(void* stream) {
  // The error word of flare_mixer_fwd_static sits at the start of the static
  // scratch, exactly where a workspace keeps it.
  void* scratch = nullptr;
  const flare_status st = static_scratch_address(&scratch);
  if (st != FLARE_OK) return st;
  return flare_last_device_status(scratch, stream);
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
