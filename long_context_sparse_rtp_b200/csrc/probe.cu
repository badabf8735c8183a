// probe.cu -- a measurement aid, not part of the layer: a kernel that keeps the
// special-function unit busy with ex2.approx.f32, so that a benchmark can time
// the device's sustained exp rate with CUDA events and quote the top-p
// selection sweeps (one exponential per (query row, causal key) pair at least)
// against it.
#include "rtp_host.h"

namespace rtp {
namespace {

constexpr int kProbeChains = 8;  // independent dependency chains per thread

__device__ __forceinline__ float ex2_probe(float x) {
  float y;
  asm volatile("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

// Every thread runs kProbeChains chains of `iters` dependent steps
// x <- ex2(-x): the values stay in (0, 1], so no step overflows or flushes.
__global__ void __launch_bounds__(256) ex2_probe_kernel(int iters, float* out) {
  float x[kProbeChains];
#pragma unroll
  for (int c = 0; c < kProbeChains; ++c) x[c] = 0.5f + 0.01f * (float)c + 1e-6f * threadIdx.x;
  for (int i = 0; i < iters; ++i) {
#pragma unroll
    for (int c = 0; c < kProbeChains; ++c) x[c] = ex2_probe(-x[c]);
  }
  float acc = 0.f;
#pragma unroll
  for (int c = 0; c < kProbeChains; ++c) acc += x[c];
  if (acc == 12345.f) out[blockIdx.x * blockDim.x + threadIdx.x] = acc;  // keeps the chains live
}

}  // namespace
}  // namespace rtp

// Launches blocks x 256 threads, each issuing iters x 8 ex2 instructions
// (blocks * 256 * iters * 8 in total).  `out` must hold blocks * 256 floats
// (it is written only in a case that never occurs).
extern "C" rtp_status rtp_probe_ex2(int32_t blocks, int32_t iters, float* out,
                                    rtp_stream_t stream) {
  if (blocks < 1 || iters < 1 || out == nullptr) return RTP_ERR_INVALID_ARG;
  rtp::ex2_probe_kernel<<<blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(iters, out);
  return rtp::check_cuda(cudaGetLastError());
}
