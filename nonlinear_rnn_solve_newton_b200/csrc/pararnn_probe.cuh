// pararnn_probe.cuh -- throughput probes: the measured peaks the solves' and the
// multi-head kernel's rooflines are reported against.
//
// The Newton solves are bound by the special-function pipe: every sigmoid and
// tanh of a cell takes one base-2 exponential and one reciprocal (ex2.approx,
// rcp.approx).  The probe runs exactly that pair, y <- 1 / (1 + 2^y), in many
// independent chains per thread at full occupancy, so the pipe, not latency,
// limits it.  y stays in (1/3, 1/2) whatever the start, so no value ever
// over- or underflows.  The second probe does the same for fp32 FMA
// (y <- y * c1 + c2, a contraction towards a fixed point), the unit the dense
// 8x8 multi-head kernel is bound by.
#pragma once

#include <cuda_runtime.h>

#include "pararnn_kernel.cuh"

namespace pararnn {

constexpr int kProbeThreads = 256;
constexpr int kProbeChains = 8;   // independent dependency chains per thread
constexpr int kProbeUnroll = 4;   // chain steps per loop trip

// PIPE 0: MUFU ex2 + rcp (2 operations per chain step); PIPE 1: fp32 FMA (1).
template <int PIPE>
__global__ void __launch_bounds__(kProbeThreads) pararnn_probe_kernel(int iters, float* sink) {
  float y[kProbeChains];
#pragma unroll
  for (int j = 0; j < kProbeChains; ++j)
    y[j] = 0.25f + 1.0e-3f * (float)((threadIdx.x + j) & 63);
  for (int i = 0; i < iters; ++i) {
#pragma unroll
    for (int u = 0; u < kProbeUnroll; ++u) {
#pragma unroll
      for (int j = 0; j < kProbeChains; ++j) {
        if constexpr (PIPE == 0) {
          y[j] = rcp_approx(1.0f + ex2_approx(y[j]));
        } else {
          y[j] = fmaf(y[j], 0.999f, 1.0e-3f);
        }
      }
    }
  }
  float s = 0.0f;
#pragma unroll
  for (int j = 0; j < kProbeChains; ++j) s += y[j];
  // never true for the values above; keeps the chains from being optimised out
  if (s == 12345.0f) sink[0] = s;
}

}  // namespace pararnn
