// pararnn_seq.cuh -- sequential application of the cells on the GPU.
//
// Two kernels, both plain applications of the recurrence h_t = f(h_{t-1}, P_t):
//   * one cell step for every channel (a decode step when generating token by
//     token; ParaRNN Figure 3 caption measures generation throughput), and
//   * the whole rollout with one thread per channel walking t = 1..L in order
//     -- the "sequential application" the parallel Newton solve is measured
//     against (ParaRNN abstract; DEER summary), here on the same GPU.
// The rollout keeps a ring of upcoming steps' inputs in flight (registers) so
// that memory latency hides behind the per-step dependency chain of the cell.
#pragma once

#include "pararnn_kernel.cuh"

namespace pararnn {

struct SeqParams {
  const void* P;      // [B, L, G, D] (rollout) or [B, G, D] (one step)
  const float* w;     // [G, D]
  const float* x0a;   // h0 (GRU) / c0 (LSTM) [B, D] or NULL
  const float* x0b;   // h0 (LSTM) or NULL
  float* out0;        // h (GRU) / c (LSTM): [B, L, D] (rollout) or [B, D] (one step)
  float* out1;        // h (LSTM)
  long long B, L, D;
};

template <int OP, typename PT>
__device__ __forceinline__ void cell_apply(const float* pin, const float* w, float* x) {
  if constexpr (OP == kGru) {
    float f, J;
    gru_cell(pin, w, x[0], f, J);
    x[0] = f;
  } else {
    float fc, fh, J[2][2];
    lstm_cell(pin, w, x[0], x[1], fc, fh, J);
    x[0] = fc;
    x[1] = fh;
  }
}

// One step for every channel: out = f(x0, P).
template <int OP, typename PT>
__global__ void __launch_bounds__(256) pararnn_step_kernel(const SeqParams p) {
  constexpr int G = OP == kGru ? 3 : 4;
  const long long n = p.B * p.D;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const long long b = i / p.D, d = i - b * p.D;
    float w[G], pin[G], x[2] = {0.0f, 0.0f};
    const PT* P = reinterpret_cast<const PT*>(p.P) + b * G * p.D + d;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      w[g] = __ldg(p.w + g * p.D + d);
      pin[g] = to_f(__ldg(P + g * p.D));
    }
    if constexpr (OP == kGru) {
      x[0] = p.x0a ? p.x0a[i] : 0.0f;
    } else {
      x[0] = p.x0a ? p.x0a[i] : 0.0f;
      x[1] = p.x0b ? p.x0b[i] : 0.0f;
    }
    cell_apply<OP, PT>(pin, w, x);
    p.out0[i] = x[0];
    if constexpr (OP == kLstm) p.out1[i] = x[1];
  }
}

// Whole rollout, one thread per channel, R steps of inputs in flight.
template <int OP, typename PT, int R>
__global__ void __launch_bounds__(128) pararnn_rollout_kernel(const SeqParams p) {
  constexpr int G = OP == kGru ? 3 : 4;
  const long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (i >= p.B * p.D) return;
  const long long b = i / p.D, d = i - b * p.D;
  float w[G];
#pragma unroll
  for (int g = 0; g < G; ++g) w[g] = __ldg(p.w + g * p.D + d);
  float x[2] = {p.x0a ? p.x0a[i] : 0.0f, 0.0f};
  if constexpr (OP == kLstm) x[1] = p.x0b ? p.x0b[i] : 0.0f;
  const PT* P = reinterpret_cast<const PT*>(p.P) + b * p.L * G * p.D + d;
  const long long step = G * p.D;  // elements between consecutive time steps
  float* o0 = p.out0 + b * p.L * p.D + d;
  float* o1 = OP == kLstm ? p.out1 + b * p.L * p.D + d : nullptr;
  // ring of the next R steps' inputs
  float ring[R][G];
#pragma unroll
  for (int s = 0; s < R; ++s)
#pragma unroll
    for (int g = 0; g < G; ++g) ring[s][g] = s < p.L ? to_f(__ldg(P + s * step + g * p.D)) : 0.0f;
  for (long long t0 = 0; t0 < p.L; t0 += R) {
#pragma unroll
    for (int s = 0; s < R; ++s) {
      const long long t = t0 + s;
      if (t < p.L) {
        float pin[G];
#pragma unroll
        for (int g = 0; g < G; ++g) pin[g] = ring[s][g];
        // refill this slot with step t + R while the cell runs
        if (t + R < p.L) {
#pragma unroll
          for (int g = 0; g < G; ++g) ring[s][g] = to_f(__ldg(P + (t + R) * step + g * p.D));
        }
        cell_apply<OP, PT>(pin, w, x);
        __stcs(o0 + t * p.D, x[0]);
        if constexpr (OP == kLstm) __stcs(o1 + t * p.D, x[1]);
      }
    }
  }
}

}  // namespace pararnn
