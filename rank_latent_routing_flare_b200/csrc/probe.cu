// Throughput probes of the two pipes the mixer's softmax runs on: the
// special-function unit (MUFU ex2.approx, one exponential per score) and the
// FP32 FMA pipe (the scale-and-shift of each score and the polynomial
// exponentials).  They give the denominators of the exp-unit roofline as
// results per SM clock, measured on the device at hand.
//
// Each CTA runs a fixed number of iterations over 8 independent dependency
// chains per thread and records (SM id, clock64 at start, clock64 at end).
// The host takes, per SM, the span from the first start to the last end of
// the CTAs that ran on it (clock64 counts that SM's own cycles) and divides
// the operations those CTAs issued by it.  The grid is one wave (a fixed
// number of CTAs per SM, all resident at once).
#include <algorithm>
#include <cstdint>
#include <vector>

#include "flare.h"
#include "flare_internal.h"

namespace flare {
namespace {

constexpr int kProbeThreads = 256;
constexpr int kProbeCtasPerSM = 4;
constexpr int kProbeChains = 8;

__device__ __forceinline__ uint32_t smid() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%smid;" : "=r"(r));
  return r;
}

// kind 0: x <- 2^(-x) on the MUFU (converges to ~0.64, never overflows)
// kind 1: x <- x * a + b on the FMA pipe
__global__ void __launch_bounds__(kProbeThreads) pipe_probe_kernel(int kind, int iters, float seed,
                                                                   unsigned long long* rec, float* sink) {
  float x[kProbeChains];
#pragma unroll
  for (int i = 0; i < kProbeChains; ++i) x[i] = seed * static_cast<float>(threadIdx.x + 1 + 37 * i);
  __syncthreads();
  const unsigned long long t0 = clock64();
  if (kind == 0) {
    for (int it = 0; it < iters; ++it) {
#pragma unroll
      for (int i = 0; i < kProbeChains; ++i) asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(x[i]) : "f"(-x[i]));
    }
  } else {
    for (int it = 0; it < iters; ++it) {
#pragma unroll
      for (int i = 0; i < kProbeChains; ++i) asm volatile("fma.rn.f32 %0, %0, %1, %2;" : "+f"(x[i]) : "f"(0.999f), "f"(1e-3f));
    }
  }
  __syncthreads();
  const unsigned long long t1 = clock64();
  float acc = 0.f;
#pragma unroll
  for (int i = 0; i < kProbeChains; ++i) acc += x[i];
  if (acc == 12345.678f) sink[0] = acc;  // keeps the chains alive; never true in practice
  if (threadIdx.x == 0) {
    rec[3 * blockIdx.x + 0] = smid();
    rec[3 * blockIdx.x + 1] = t0;
    rec[3 * blockIdx.x + 2] = t1;
  }
}

// Results per clock per SM of one probe kind, from the CTA records.
double rate_per_clk_sm(const std::vector<unsigned long long>& rec, int nblocks, double ops_per_block) {
  std::vector<unsigned long long> lo(1024, ~0ull), hi(1024, 0ull);
  std::vector<int> cnt(1024, 0);
  for (int b = 0; b < nblocks; ++b) {
    const unsigned long long s = rec[3 * b];
    if (s >= 1024) continue;
    lo[s] = std::min(lo[s], rec[3 * b + 1]);
    hi[s] = std::max(hi[s], rec[3 * b + 2]);
    ++cnt[s];
  }
  double sum = 0.0;
  int n = 0;
  for (int s = 0; s < 1024; ++s) {
    if (cnt[s] == 0 || hi[s] <= lo[s]) continue;
    sum += cnt[s] * ops_per_block / static_cast<double>(hi[s] - lo[s]);
    ++n;
  }
  return n > 0 ? sum / n : 0.0;
}

}  // namespace
}  // namespace flare

using namespace flare;

extern "C" {

size_t flare_probe_scratch_bytes(void) {
  return static_cast<size_t>(kNumSM) * kProbeCtasPerSM * 3 * sizeof(unsigned long long) + 256;
}

flare_status flare_probe_pipe_rates(void* scratch, size_t scratch_bytes, void* stream, double* ex2_per_clk_sm,
                                    double* ffma_per_clk_sm) {
  if (!scratch || !ex2_per_clk_sm || !ffma_per_clk_sm) return FLARE_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(scratch) & 255u) != 0) return FLARE_ERR_ALIGN;
  if (scratch_bytes < flare_probe_scratch_bytes()) return FLARE_ERR_WORKSPACE;
  int dev = 0, nsm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return FLARE_ERR_LAUNCH;
  nsm = std::min(nsm, kNumSM);
  const int nblocks = nsm * kProbeCtasPerSM;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  auto* rec = static_cast<unsigned long long*>(scratch);
  float* sink = reinterpret_cast<float*>(static_cast<uint8_t*>(scratch) + flare_probe_scratch_bytes() - 256);
  std::vector<unsigned long long> host(3 * static_cast<size_t>(nblocks));
  const int iters[2] = {2048, 8192};
  double out[2] = {0.0, 0.0};
  for (int kind = 0; kind < 2; ++kind) {
    for (int rep = 0; rep < 2; ++rep) {  // the first run warms the clocks up
      pipe_probe_kernel<<<nblocks, kProbeThreads, 0, s>>>(kind, iters[kind], 1e-3f, rec, sink);
      if (cudaGetLastError() != cudaSuccess) return FLARE_ERR_LAUNCH;
    }
    if (cudaMemcpyAsync(host.data(), rec, host.size() * sizeof(unsigned long long), cudaMemcpyDeviceToHost, s) !=
            cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
      return FLARE_ERR_LAUNCH;
    out[kind] = rate_per_clk_sm(host, nblocks, static_cast<double>(kProbeThreads) * iters[kind] * kProbeChains);
  }
  *ex2_per_clk_sm = out[0];
  *ffma_per_clk_sm = out[1];
  return FLARE_OK;
}

}  // extern "C"
