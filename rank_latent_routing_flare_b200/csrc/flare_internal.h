// Internal definitions shared by the FLARE kernels and the host entry points.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

// Device error word bits (first 4 bytes of the workspace).
#define FLARE_DEV_TIMEOUT 0x1u
#define FLARE_DEV_BAD_LENGTH 0x2u
#define FLARE_DEV_UNDERFLOW 0x4u   // a merged row lost mass and could not be recomputed exactly
#define FLARE_DEV_NO_STATE 0x8u    // a backward that reuses a training forward's state found none

namespace flare {

// Valid tokens of sequence b within one shard: `lengths` (NULL = all valid)
// counts tokens of the whole sequence of n_global tokens, and the shard holds
// tokens [tok_offset, tok_offset + N).  A length outside [1, n_global] is
// clamped; *bad is set.
__host__ __device__ inline int shard_valid_len(const int32_t* lengths, int b, int N, int tok_offset, int n_global,
                                               bool* bad) {
  if (lengths == nullptr) return N;
  int l = lengths[b];
  if (l < 1 || l > n_global) {
    *bad = true;
    l = l < 0 ? 0 : (l > n_global ? n_global : l);
  }
  l -= tok_offset;
  return l < 0 ? 0 : (l > N ? N : l);
}

constexpr int kNumSM = 148;        // B200
constexpr int kLatBlock = 128;     // latents per encode CTA (UMMA M)
constexpr int kDecTile = 128;      // tokens per decode tile (UMMA M)
constexpr int kNormGroup = 32;     // tokens per key-norm group
constexpr int kProjTile = 128;     // tokens per projection tile

// Tokens per encoder tile and score buffers in TMEM.  The encoder keeps
// enc_bufs score tiles and the output accumulator (D + 16 columns) in TMEM:
// 2 * 48 + 32 = 128 columns for D = 16 (four CTAs per SM), and 3 * 64 + 48
// (within 256, two CTAs per SM) for D = 32.  Chosen by measurement on B200:
// at D = 16 three 32-token buffers (the same 128 columns) were 12 % slower
// than two 48-token ones.
#ifndef FLARE_ENC_TILE_D16
#define FLARE_ENC_TILE_D16 48
#endif
#ifndef FLARE_ENC_BUFS_D16
#define FLARE_ENC_BUFS_D16 2
#endif
#ifndef FLARE_ENC_BUFS_D32
#define FLARE_ENC_BUFS_D32 3
#endif
__host__ __device__ constexpr int enc_tile(int D) { return D == 16 ? FLARE_ENC_TILE_D16 : 64; }
__host__ __device__ constexpr int enc_bufs(int D) { return D == 16 ? FLARE_ENC_BUFS_D16 : FLARE_ENC_BUFS_D32; }
// Co-resident CTAs per SM of the encoder: 128 TMEM columns per CTA for
// D = 16 (up to four CTAs), 256 for D = 32 (two).
#ifndef FLARE_ENC_CTAS_D16
#define FLARE_ENC_CTAS_D16 4
#endif
__host__ __device__ constexpr int enc_ctas_per_sm(int D) { return D == 16 ? FLARE_ENC_CTAS_D16 : 2; }
// Latents per decoder chunk and score buffers, as for the encoder: 2 * 48
// + 32 = 128 TMEM columns for D = 16, 3 * 64 + 48 (within 256) for D = 32.
#ifndef FLARE_DEC_CHUNK_D16
#define FLARE_DEC_CHUNK_D16 48
#endif
#ifndef FLARE_DEC_BUFS_D16
#define FLARE_DEC_BUFS_D16 2
#endif
#ifndef FLARE_DEC_BUFS_D32
#define FLARE_DEC_BUFS_D32 3
#endif
__host__ __device__ constexpr int dec_chunk(int D) { return D == 16 ? FLARE_DEC_CHUNK_D16 : 64; }
__host__ __device__ constexpr int dec_bufs(int D) { return D == 16 ? FLARE_DEC_BUFS_D16 : FLARE_DEC_BUFS_D32; }
// Co-resident CTAs per SM of the decoder (TMEM columns as for the encoder).
#ifndef FLARE_DEC_CTAS_D16
#define FLARE_DEC_CTAS_D16 4
#endif
__host__ __device__ constexpr int dec_ctas_per_sm(int D) { return D == 16 ? FLARE_DEC_CTAS_D16 : 2; }

// Of every 32 score pairs of a softmax row, how many are exponentiated on
// the FMA pipe (polynomial, paired fp32 instructions) instead of the MUFU;
// chosen by measurement on B200.
#ifndef FLARE_ENC_POLY_PAIRS
#define FLARE_ENC_POLY_PAIRS 11
#endif
// Encoder softmax: load the first 16 score columns, start their
// exponentials while the rest of the tile is read from TMEM.
#ifndef FLARE_ENC_SPLIT_LD
#define FLARE_ENC_SPLIT_LD 1
#endif
// Heads (D = 16; half as many for D = 32) whose projection outputs are read
// from TMEM per wait.
#ifndef FLARE_PROJ_EPI_HEADS
#define FLARE_PROJ_EPI_HEADS 4
#endif
#ifndef FLARE_DEC_POLY_PAIRS
#define FLARE_DEC_POLY_PAIRS 10
#endif

// ---------------------------------------------------------------------------
// Projection: out[p][b][h][n][:] = X[b][n][:] @ W_p[:, h*D:(h+1)*D]
// ---------------------------------------------------------------------------
struct ProjParams {
  int B, N, C, H, D;
  int tiles_per_b;     // ceil(N / kProjTile)
  int n_tiles;         // B * tiles_per_b
  int groups;          // CTAs per projection
  int n_groups32;      // ceil(N / kNormGroup)
  int n_proj;          // projections computed: 1, 2 or 4 (weights tm_w0 .. tm_w{n_proj-1})
  int token_major;     // 0: out [B][H][N][D]; 1: out [B][N][C] (row n = heads side by side)
  uint16_t* out[4];    // bf16, layout per token_major
  float* knorm[4];     // [B*H][n_groups32] max key norm per group, or nullptr
  uint32_t* err;
  unsigned long long timeout_ns;
};

// ---------------------------------------------------------------------------
// Key norms for the FLARE path (keys given by the caller)
// ---------------------------------------------------------------------------
struct KnormParams {
  int BH, N, D, n_groups32;
  const uint16_t* k;   // [BH][N][D]
  float* knorm;        // [BH][n_groups32]
};

// ---------------------------------------------------------------------------
// Split-N encode: partial softmax sums of one (b, h, latent block, split)
// ---------------------------------------------------------------------------
struct EncodeParams {
  int B, H, N, M, D;
  int q_per_batch;      // queries [B*H][M][D] (1) or [H][M][D] (0)
  int n_splits;         // S
  int tiles_per_split;  // in tiles of enc_tile(D) tokens
  int n_lblocks;        // ceil(M / kLatBlock)
  int n_groups32;
  int q_rows;           // rows of one query box: min(M, kLatBlock)
  int tok_offset;       // first token of this shard (context parallelism; else 0)
  int n_global;         // tokens of the whole sequence (else N)
  float c;              // scale * log2(e)
  const int32_t* lengths;
  const float* knorm;   // [B*H][n_groups32]
  const uint16_t* q;    // bf16 queries
  float* part;          // [B*H][S][M][D+2]: shift, sum, D partial outputs
  uint32_t* err;
  unsigned long long timeout_ns;
};

// ---------------------------------------------------------------------------
// Merge of the split partials (log-sum-exp combine) + exact fallback rows
// ---------------------------------------------------------------------------
struct MergeParams {
  int B, H, N, M, D;    // N: tokens of one shard (of the sequence without context parallelism)
  int q_per_batch;
  int n_splits, tiles_per_split;
  int n_ranks;          // shards whose partials are merged (1 without context parallelism)
  int allow_exact;      // rows whose sums underflowed: recompute from q, k, v (1) or report (0)
  size_t rank_stride;   // floats between the partials of consecutive shards
  uint32_t* err;
  float scale, c;
  const int32_t* lengths;
  const float* part;
  const uint16_t* q;    // bf16 queries of this encode
  const uint16_t* k;    // bf16 keys   [B*H][N][D]
  const uint16_t* v;    // bf16 values [B*H][N][D]
  float* out_f32;       // [B*H][M][D]
  uint16_t* out_bf16;   // [B*H][M][D]
  const float* fix;     // context parallelism: every shard's exact partials of the rows that need
                        // them, [n_ranks][B*H*M][D+2] rank-major, or nullptr
  size_t fix_rank_stride;  // floats between consecutive shards' exact partials
  float* lse_out;       // optional [B*H][M]: L_m = log2 sum_n 2^(c <q_m, k_n>), the row's log-normaliser
};

// ---------------------------------------------------------------------------
// Decode: Y = softmax_m(K Q^T * scale) Z per token
// ---------------------------------------------------------------------------
struct DecodeParams {
  int B, H, N, M, D;
  int q_per_batch;
  int tiles_per_cta;    // in kDecTile tiles
  int tok_offset;       // first token of this shard (context parallelism; else 0)
  int n_global;         // tokens of the whole sequence (else N)
  int ctas_per_head;
  int qz_box_rows;      // rows of one Q/Z box: min(M, 256)
  float scale, c;
  const int32_t* lengths;
  const uint16_t* q;    // bf16 [G][M][D]
  const uint16_t* z;    // bf16 [B*H][M][D]
  const uint16_t* k;    // bf16 [B*H][N][D]
  uint16_t* y;          // bf16 [B*H][N][D], or [B][N][H*D] when y_token_major; null: not stored
  int y_token_major;
  float* y_f32;         // optional fp32 copy of Y ([B*H][N][D], the values Y is rounded from), or nullptr
  // the training forward's variant (D = 16): z holds fp16 bits of Z and the
  // softmax weights enter the value product in fp16 (scaled by 2^14), so
  // that Y sees Z to 2^-12; the exact fallback takes z32 (fp32 Z)
  int z_f16;
  const float* z32;
  float* ltok_out;      // optional [B*H][N]: L_n = log2 sum_m 2^(c <k_n, q_m>) per token (0 for padding)
  uint32_t* fb_count;   // number of listed tokens (zeroed before the decoder runs)
  uint64_t* fb_list;    // tokens (bh * N + n) whose row sum underflowed, capacity B*H*N
  uint32_t* err;
  unsigned long long timeout_ns;
};

// Launch configuration of one kernel.  With pdl (programmatic dependent
// launch) the kernel may begin -- its CTAs become resident and run their
// set-up -- while the previous kernel on the stream is still finishing; every
// kernel of this library calls pdl_wait() before its first access to global
// memory that another kernel writes or reads, and calls
// pdl_launch_dependents() early so that the next kernel can start.  Only a
// kernel whose predecessor on the stream is a kernel of the same call is
// launched with pdl.
struct LaunchCfg {
  cudaLaunchConfig_t cfg{};
  cudaLaunchAttribute attr[1];
  LaunchCfg(dim3 grid, dim3 block, size_t smem, cudaStream_t s, bool pdl) {
#ifdef FLARE_NO_PDL
    pdl = false;
#endif
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = pdl ? attr : nullptr;
    cfg.numAttrs = pdl ? 1 : 0;
  }
};

// Host-side launchers (each returns the cudaError_t of the launch; pdl as
// for LaunchCfg).
cudaError_t launch_project(const CUtensorMap& tm_x, const CUtensorMap (&tm_w)[4], const ProjParams& p,
                           cudaStream_t s, bool pdl = false);
cudaError_t launch_knorm(const KnormParams& p, cudaStream_t s);
cudaError_t launch_encode(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                          const EncodeParams& p, cudaStream_t s, bool pdl = false);
cudaError_t launch_merge(const MergeParams& p, cudaStream_t s, bool pdl = false);
// dst[i] = fp16(src[i]) for i < n (n even).
struct ToF16Params {
  long n;
  const float* src;
  uint16_t* dst;
};
cudaError_t launch_to_f16(const ToF16Params& p, cudaStream_t s);
cudaError_t launch_cp_exact(const MergeParams& p, int rank, float* out, cudaStream_t s);
cudaError_t launch_decode(const CUtensorMap& tm_q, const CUtensorMap& tm_z, const CUtensorMap& tm_k,
                          const DecodeParams& p, cudaStream_t s, bool pdl = false);
cudaError_t launch_wait_selftest(uint32_t* err, unsigned long long timeout_ns, cudaStream_t s);

// Shared-memory footprints (bytes) of the pipelined kernels.
size_t encode_smem_bytes(int D);
size_t decode_smem_bytes(int D);
size_t project_smem_bytes(int C);

}  // namespace flare
