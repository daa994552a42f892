// pararnn_seq.cuh -- sequential application of the cells on the GPU.
//
// Two kernels, both plain applications of the recurrence h_t = f(h_{t-1}, P_t):
//   * one cell step for every channel (a decode step when generating token by
//     token; ParaRNN Figure 3 caption measures generation throughput), and
//   * the whole rollout with one thread per channel walking t = 1..L in order
//     -- the "sequential application" the parallel Newton solve is measured
//     against (ParaRNN abstract; DEER summary), here on the same GPU.
// When a warp's 32 threads hold 32 consecutive channels of one batch row (D a
// multiple of 32), the rollout stages its inputs through shared memory: the
// warp copies the next R steps' rows of its channels with cp.async into one of
// two buffers while it applies the cell to the current R steps, and waits for
// the copy groups one at a time.  Loads kept in registers instead (the
// fallback for other D) are waited for in batches by the hardware, so in
// practice each step waits for a memory round trip.
#pragma once

#include "pararnn_kernel.cuh"
#include "pararnn_walk.cuh"

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

// One warp's copy of R steps x G gate rows of its 32 channels (one 16-byte
// chunk per lane and round) into dst[R][G][32]; steps at or past L are zero-filled.
template <typename PT, int G, int R>
__device__ __forceinline__ void stage_rows(PT* dst, const PT* src, long long t_first,
                                           long long L, long long D, int lane) {
  constexpr int CPR = 32 * (int)sizeof(PT) / 16;  // 16-byte chunks per row
  constexpr int NCH = R * G * CPR;
#pragma unroll
  for (int k = lane; k < NCH; k += 32) {
    const int s = k / (G * CPR), g = (k / CPR) % G, c = k % CPR;
    const long long t = t_first + s;
    const bool valid = t < L;
    const PT* row = src + ((valid ? t : 0) * G + g) * D;
    cp_async16(smem_u32(dst + (s * G + g) * 32) + 16u * c,
               reinterpret_cast<const char*>(row) + 16 * c, valid);
  }
  cp_async_commit();
}

// The rollout above with staged inputs: 4 warps per CTA, each on 32 consecutive
// channels of one batch row (requires D % 32 == 0 and P 16-byte aligned).
template <int OP, typename PT, int R>
__global__ void __launch_bounds__(128) pararnn_rollout_staged_kernel(const SeqParams p) {
  constexpr int G = OP == kGru ? 3 : 4;
  __shared__ __align__(16) PT s_in[4][2][R * G * 32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (i >= p.B * p.D) return;  // whole warps: B D is a multiple of 32
  const long long b = i / p.D, d = i - b * p.D;
  float w[G];
#pragma unroll
  for (int g = 0; g < G; ++g) w[g] = __ldg(p.w + g * p.D + d);
  float x[2] = {p.x0a ? p.x0a[i] : 0.0f, 0.0f};
  if constexpr (OP == kLstm) x[1] = p.x0b ? p.x0b[i] : 0.0f;
  const PT* P = reinterpret_cast<const PT*>(p.P) + b * p.L * G * p.D + (d - lane);
  float* o0 = p.out0 + b * p.L * p.D + d;
  float* o1 = OP == kLstm ? p.out1 + b * p.L * p.D + d : nullptr;
  PT* buf0 = s_in[warp][0];
  PT* buf1 = s_in[warp][1];
  stage_rows<PT, G, R>(buf0, P, 0, p.L, p.D, lane);
  stage_rows<PT, G, R>(buf1, P, R, p.L, p.D, lane);
  for (long long t0 = 0, blk = 0; t0 < p.L; t0 += R, ++blk) {
    PT* buf = (blk & 1) ? buf1 : buf0;
    cp_async_wait_prior();  // this buffer's group has landed
    __syncwarp();
#pragma unroll
    for (int s = 0; s < R; ++s) {
      const long long t = t0 + s;
      if (t < p.L) {
        float pin[G];
#pragma unroll
        for (int g = 0; g < G; ++g) pin[g] = to_f(buf[(s * G + g) * 32 + lane]);
        cell_apply<OP, PT>(pin, w, x);
        __stcs(o0 + t * p.D, x[0]);
        if constexpr (OP == kLstm) __stcs(o1 + t * p.D, x[1]);
      }
    }
    __syncwarp();  // every lane has read this buffer
    stage_rows<PT, G, R>(buf, P, t0 + 2 * R, p.L, p.D, lane);
  }
  cp_async_wait_all();
}

// The rollout for one channel per batch row (D = 1, the DEER shape): a
// thread's sequence is one contiguous run of L x G inputs, so each thread
// copies its own next R steps (R G elements, a multiple of 16 bytes) with
// cp.async into one of two buffers.  Requires P 16-byte aligned and
// L G sizeof(PT) a multiple of 16.
template <int OP, typename PT, int R>
__global__ void __launch_bounds__(64) pararnn_rollout_seq1_kernel(const SeqParams p) {
  constexpr int G = OP == kGru ? 3 : 4;
  constexpr int CH = R * G * (int)sizeof(PT) / 16;  // 16-byte chunks per group
  static_assert((R * G * sizeof(PT)) % 16 == 0, "whole 16-byte chunks");
  __shared__ __align__(16) PT s_in[64][2][R * G];
  const long long b = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (b >= p.B) return;
  float w[G];
#pragma unroll
  for (int g = 0; g < G; ++g) w[g] = __ldg(p.w + g);
  float x[2] = {p.x0a ? p.x0a[b] : 0.0f, 0.0f};
  if constexpr (OP == kLstm) x[1] = p.x0b ? p.x0b[b] : 0.0f;
  const char* src = reinterpret_cast<const char*>(reinterpret_cast<const PT*>(p.P) + b * p.L * G);
  const long long nbytes = p.L * G * (long long)sizeof(PT);
  float* o0 = p.out0 + b * p.L;
  float* o1 = OP == kLstm ? p.out1 + b * p.L : nullptr;
  PT* const buf0 = s_in[threadIdx.x][0];
  PT* const buf1 = s_in[threadIdx.x][1];
  auto stage = [&](PT* dst, long long t_first) {
    const long long off = t_first * G * (long long)sizeof(PT);
#pragma unroll
    for (int k = 0; k < CH; ++k) {
      const long long o = off + 16 * k;
      const bool valid = o < nbytes;  // nbytes is a multiple of 16
      cp_async16(smem_u32(dst) + 16u * k, src + (valid ? o : 0), valid);
    }
    cp_async_commit();
  };
  stage(buf0, 0);
  stage(buf1, R);
  for (long long t0 = 0, blk = 0; t0 < p.L; t0 += R, ++blk) {
    PT* cur = (blk & 1) ? buf1 : buf0;
    cp_async_wait_prior();
#pragma unroll
    for (int s = 0; s < R; ++s) {
      const long long t = t0 + s;
      if (t < p.L) {
        float pin[G];
#pragma unroll
        for (int g = 0; g < G; ++g) pin[g] = to_f(cur[s * G + g]);
        cell_apply<OP, PT>(pin, w, x);
        __stcs(o0 + t, x[0]);
        if constexpr (OP == kLstm) __stcs(o1 + t, x[1]);
      }
    }
    stage(cur, t0 + 2 * R);
  }
  cp_async_wait_all();
}

// Multi-head GRU (dense 8x8 blocks per head of 8 channels) applied in order:
// 8 lanes per (batch row, head) sequence, lane i = channel i of the head.  Per
// step the head's state is gathered from the group by shuffles, lane i forms
// row i of U_z h, U_r h and U_c h, and
//   z = sig(P_z + U_z h), r = sig(P_r + U_r h), c = tanh(P_c + r (U_c h)),
//   h' = (1 - z) h + z c.
// A ring of the next R steps' inputs stays in flight, as in the rollout above.
struct MhSeqParams {
  const void* P;   // [B, L, 3, D], D = 8 H
  const float* U;  // [3, H, 8, 8]: gate, head, row, column
  const float* h0; // [B, D] or NULL
  float* h;        // [B, L, D]
  long long B, L, H;
};

template <typename PT, int R, bool STAGED>
__global__ void __launch_bounds__(64) pararnn_rollout_mhgru_kernel(const MhSeqParams p) {
  const long long gid = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  const long long seq = gid >> 3;  // (batch row, head); the 8 lanes of a group agree
  if (seq >= p.B * p.H) return;
  const int i = threadIdx.x & 7;
  const unsigned gmask = 0xffu << (threadIdx.x & 24);
  const long long b = seq / p.H, g = seq - b * p.H;
  const long long D = 8 * p.H;
  float uz[8], ur[8], uc[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    uz[j] = __ldg(p.U + ((0 * p.H + g) * 8 + i) * 8 + j);
    ur[j] = __ldg(p.U + ((1 * p.H + g) * 8 + i) * 8 + j);
    uc[j] = __ldg(p.U + ((2 * p.H + g) * 8 + i) * 8 + j);
  }
  const long long ch = b * D + 8 * g + i;
  float h = p.h0 ? __ldg(p.h0 + ch) : 0.0f;
  const PT* P = reinterpret_cast<const PT*>(p.P) + b * p.L * 3 * D + 8 * g + i;
  const long long step = 3 * D;
  float* out = p.h + b * p.L * D + 8 * g + i;
  // staged: this warp's 32 channels (4 heads) through shared memory
  __shared__ __align__(16) PT s_in[STAGED ? 2 : 1][2][STAGED ? R * 3 * 32 : 1];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const PT* Pw = P - lane;  // staged: the warp's first channel (D % 32 == 0: one batch row)
  float ring[STAGED ? 1 : R][3];
  if constexpr (STAGED) {
    stage_rows<PT, 3, R>(s_in[warp][0], Pw, 0, p.L, D, lane);
    stage_rows<PT, 3, R>(s_in[warp][1], Pw, R, p.L, D, lane);
  } else {
#pragma unroll
    for (int s = 0; s < R; ++s)
#pragma unroll
      for (int q = 0; q < 3; ++q) ring[s][q] = s < p.L ? to_f(__ldg(P + s * step + q * D)) : 0.0f;
  }
  for (long long t0 = 0, blk = 0; t0 < p.L; t0 += R, ++blk) {
    PT* buf = s_in[STAGED ? warp : 0][blk & 1];
    if constexpr (STAGED) {
      cp_async_wait_prior();
      __syncwarp();  // every lane's copies of this buffer are visible
    }
#pragma unroll
    for (int s = 0; s < R; ++s) {
      const long long t = t0 + s;
      if (t < p.L) {
        float pz, pr, pc;
        if constexpr (STAGED) {
          pz = to_f(buf[(s * 3 + 0) * 32 + lane]);
          pr = to_f(buf[(s * 3 + 1) * 32 + lane]);
          pc = to_f(buf[(s * 3 + 2) * 32 + lane]);
        } else {
          pz = ring[s][0], pr = ring[s][1], pc = ring[s][2];
          if (t + R < p.L) {
#pragma unroll
            for (int q = 0; q < 3; ++q) ring[s][q] = to_f(__ldg(P + (t + R) * step + q * D));
          }
        }
        float az = pz, ar = pr, ac = 0.0f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float hj = __shfl_sync(gmask, h, j, 8);
          az = fmaf(uz[j], hj, az);
          ar = fmaf(ur[j], hj, ar);
          ac = fmaf(uc[j], hj, ac);
        }
        const float z = sigm(az);
        const float r = sigm(ar);
        const float c = tanh_f(fmaf(r, ac, pc));
        h = fmaf(z, c - h, h);
        __stcs(out + t * D, h);
      }
    }
    if constexpr (STAGED) {
      __syncwarp();  // every lane has read this buffer
      stage_rows<PT, 3, R>(buf, Pw, t0 + 2 * R, p.L, D, lane);
    }
  }
  if constexpr (STAGED) cp_async_wait_all();
}

}  // namespace pararnn
