// Host-side definitions shared by the C-ABI translation units (api.cu: the
// forward and its context-parallel phases; api_bwd.cu: the backward).
#pragma once

#include <cstddef>
#include <cstdint>

#include "flare.h"
#include "flare_internal.h"

namespace flare {

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Tensor maps (api.cu): bf16 3-D [d2][d1][d0] with box (b0, b1, 1); fp32 2-D
// [d1][d0] with box (b0, b1); the row swizzle of a D-wide bf16 operand.
bool map3d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t b0, uint32_t b1,
           CUtensorMapSwizzle sw);
bool map2d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint32_t b0, uint32_t b1,
           CUtensorMapSwizzle sw);
bool map2d_f32(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint32_t b0, uint32_t b1);
CUtensorMapSwizzle row_swizzle(int D);
unsigned long long wait_timeout_ns();
inline long cdiv(long a, long b) { return (a + b - 1) / b; }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The first bytes of every workspace: the device error word (offset 0), the
// decoder's fallback counter (4) and the training forward's mark (8).  Every
// entry point but the training backward clears all three when it starts, so
// that any other call in a workspace invalidates a training forward's state;
// the training backward clears only the first two (kErrWordBytes) and checks
// the mark on the device.
constexpr size_t kErrWordBytes = 8;
constexpr size_t kTrainMarkOffset = 8;
constexpr size_t kErrClearBytes = 16;

// Workspace layout and launch shapes of the forward.
struct Plan {
  int S = 1, tps = 1, LB = 1;            // encoder splits, tiles per split, latent blocks
  int dec_ctas = 1, dec_tiles = 1;       // decoder CTAs per head, tiles per CTA
  int G32 = 1;
  size_t off_err = 0, off_kt = 0, off_vt = 0, off_kp = 0, off_vp = 0, off_kn_syn = 0, off_kn = 0, off_part = 0,
         off_qx32 = 0, off_qx16 = 0, off_z32 = 0, off_z16 = 0, off_fb = 0, off_ycat = 0, total = 0;
};

Plan make_plan(int variant, long B, long H, long N, long M, long D);

// Workspace of the backward: the forward's (projection outputs, error word)
// followed by the fp32 recompute and gradient buffers.
struct BwdPlan {
  Plan fwd;
  int S = 1, tps = 1, rpb = 32, LB = 1, dw_splits = 1;
  size_t off_q32 = 0, off_qx32 = 0, off_lsyn = 0, off_dqx32 = 0, off_gsyn = 0, off_z32 = 0, off_lenc = 0,
         off_ltok = 0, off_dtok = 0, off_dz32 = 0, off_gam = 0, off_fpart = 0, off_pa = 0, off_pc = 0,
         off_grows = 0, off_dwpart = 0, off_y32 = 0, off_zf16 = 0, off_xhi16 = 0, off_xlo16 = 0, off_zhi16 = 0, off_zlo16 = 0, off_qpad = 0, off_q0pad = 0, off_zpad = 0, off_dzpad = 0,
         off_dqxpad = 0, off_dqxdec = 0, total = 0;
};

BwdPlan make_bwd_plan(bool pp, long B, long H, long N, long M, long D, long C);

// Number of token splits of a split-N pass (the encoder's wave cost model;
// setup_tiles: a CTA's fixed cost in tiles of work).
int choose_splits(long units, long ntiles, long slots, long setup_tiles);

flare_status check_common(int B, int H, int N, int M, int D);
float resolve_scale(float scale, int D);
flare_status check_flarepp(const void* X, const void* Wk, const void* Wv, const void* Wk_syn, const void* Wv_syn,
                           const void* Q0, const void* Y, int B, int N, int C, int H, int M, int D,
                           const int32_t* lengths, const void* workspace, const float* Qx_out, const float* Z_out);

// Statistics a training forward leaves for the backward (each optional):
// the row log-normalisers of the synthesis and the encode ([B*H][M]), in
// log2 units; and, with zf16 (D = 16), where the decoder's fp16 copy of Z
// goes (its value product then runs in fp16, so that Y sees Z to 2^-12), the
// fp32 Y and the decoder's per-token log-normalisers ([B*H][N]).
struct FwdStats {
  float *lsyn = nullptr, *lenc = nullptr;
  uint16_t* zf16 = nullptr;
  float *y32 = nullptr, *ltok = nullptr;
};

// The FLARE forward (eq. 5-6) and the FLARE++ pipeline (eq. 7-11) after the
// argument checks of their entry points; Y_f32_out and stats are optional.
flare_status flare_fwd(const flare_bf16* K, const flare_bf16* V, const flare_bf16* Q, flare_bf16* Y, int B, int H,
                       int N, int M, int D, const int32_t* lengths, float scale, void* workspace,
                       size_t workspace_bytes, void* stream, float* Z_out, float* Y_f32_out,
                       void* const* stage_events, const FwdStats* stats);
flare_status flarepp_run(const Plan& pl, const flare_bf16* X, const flare_bf16* Wk, const flare_bf16* Wv,
                         const flare_bf16* Wk_syn, const flare_bf16* Wv_syn, const flare_bf16* Q0, void* Y,
                         int y_token_major, int B, int N, int C, int H, int M, int D, const int32_t* lengths,
                         float sc, uint8_t* ws, cudaStream_t s, float* Qx_out, float* Z_out,
                         void* const* stage_events, float* Y_f32_out, const FwdStats* stats);

// Outputs of the FLARE++ projections in the workspace.
struct Projected {
  uint16_t *kt, *vt, *kk, *vv;
  float *kn_syn, *kn;
};

// eq. 7 and eq. 9: the per-head projections of X into the workspace (two
// when the synthesis and encode weights are the same tensors, else four).
flare_status flarepp_project(const Plan& pl, const flare_bf16* X, const flare_bf16* Wk, const flare_bf16* Wv,
                             const flare_bf16* Wk_syn, const flare_bf16* Wv_syn, int B, int N, int C, int H, int D,
                             uint8_t* ws, cudaStream_t s, void* const* stage_events, Projected* pr);

}  // namespace flare
