// pararnn_mhgru2.cuh -- the multi-head GRU Newton solve (dense 8x8 recurrence
// blocks) with a head's 8 channels spread over 8 lanes.
//
// Same method, cell and stopping rule as pararnn_mhgru.cuh (DEER summary,
// caveats: dense Jacobians, O(n^3) per step with n = 8 per head), organised for
// occupancy.  Keeping a whole 8x8 segment map and an 8x8 Jacobian in one lane
// takes ~250 registers, and one warp per (batch row, head) sequence leaves only
// ~7 warps per SM at 1024 sequences.  Here:
//   * a group of 8 lanes owns one time segment of S steps of one sequence; lane
//     i evaluates row i of the cell (its gates z_i, r_i, c_i, f_i, the residual)
//     and row i of the Jacobian, and keeps column i of the segment's running map
//     A = J_t ... J_1 (and component i of its offset b);
//   * per step the 8 Jacobian rows meet in shared memory, and lane i updates its
//     column, A[:, i] <- J A[:, i], and its offset component,
//     b_i <- (J b)_i + bt_i (bt = f - J h^k_{t-1}, the map's offset);
//   * a CTA of MW warps = 4 MW groups walks one sequence: its chunk is 4 MW
//     consecutive segments; one group then carries the chunk's incoming state
//     through the segment maps (x_{k+1} = A_k x_k + b_k, a matrix-vector product
//     per segment shared by the group's 8 lanes), and every group applies its
//     steps from its segment's incoming state, recomputing the cell rows:
//     h^{k+1}_t = f_t + J_t (h^{k+1}_{t-1} - h^k_{t-1});
//   * CTAs are persistent (cooperative launch); Newton iterations are separated
//     by a grid barrier and the global max-abs residual, as for every solve here.
// Time strides (one per head) are handled as in pararnn_mhgru.cuh: a unit is
// (batch row, head, residue r) and its position k is time step r + k s.
#pragma once

#include "pararnn_kernel.cuh"
#include "pararnn_mhgru.cuh"

#ifndef PARARNN_MH2_WARPS
#define PARARNN_MH2_WARPS 2
#endif
// Steps per segment, measured on B200 (B=8, L=4096, 128 heads, fp32): 8 steps
// 3.17 ms unstrided / 5.42 ms with strides 2^(g mod 8); 16 steps 3.05 / 5.99 ms;
// 32 steps 4.68 / 8.65 ms; 4 warps per CTA (16 steps) 3.75 / 6.49 ms.
#ifndef PARARNN_MH2_STEPS
#define PARARNN_MH2_STEPS 8
#endif

namespace pararnn {

constexpr int kMh2Warps = PARARNN_MH2_WARPS;
constexpr int kMh2S = PARARNN_MH2_STEPS;          // steps per segment
constexpr int kMh2Seg = 4 * kMh2Warps;            // segments (groups) per CTA
constexpr int kMh2T = kMh2Seg * kMh2S;            // steps per chunk
constexpr int kMh2Threads = 32 * kMh2Warps;

// Shared-memory rows are grouped by segment, with a pad after each segment's
// block: the 4 groups of a warp read the same step of 4 consecutive segments at
// once, and without the pad those rows would sit a multiple of 32 words apart
// (the same banks).  The pads put the groups 8 words apart.
constexpr int kMh2HkSeg = kMh2S * 8 + 8;      // floats per segment block of h^k rows
constexpr int kMh2GateSeg = kMh2S * 24 + 8;   // elements per segment block of gate rows
constexpr int kMh2JStride = 64 + 4;           // floats per group's Jacobian block
static_assert((kMh2GateSeg * 2) % 16 == 0, "bf16 gate rows stay 16-byte aligned");

// h^k row of chunk position t (-1 = the step before the chunk), gate row of t
__device__ __forceinline__ int mh2_hk(int t) {
  return t < 0 ? 0 : 8 + (t / kMh2S) * kMh2HkSeg + (t % kMh2S) * 8;
}
__device__ __forceinline__ int mh2_gate(int t) {
  return (t / kMh2S) * kMh2GateSeg + (t % kMh2S) * 24;
}

template <typename PT> struct Mh2Smem {
  float hk[8 + kMh2Seg * kMh2HkSeg];      // h^k: the step before the chunk, then per segment
  PT gates[kMh2Seg * kMh2GateSeg];        // the chunk's P: per step z[8], r[8], c[8]
  float J[kMh2Seg][kMh2JStride];          // per group: the current step's Jacobian rows
  float A[kMh2Seg][8][8];           // per segment: its map, by columns (A[k][col][row])
  float bv[kMh2Seg][8];             // per segment: its map's offset
  float xin[kMh2Seg + 1][8];        // the state entering each segment (+ leaving the chunk)
  float U[3][8][8];                 // the head's blocks (gate, row, column)
};

// Row i of the cell at h (U row i of each gate; gates z_i, r_i, c_i): returns
// f_i and writes row i of the Jacobian.
__device__ __forceinline__ float mh2_row(const float* h, const float* uz, const float* ur,
                                         const float* uc, float pz, float pr, float pc, int i,
                                         float* Jrow) {
  float az = 0.0f, ar = 0.0f, ac = 0.0f;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    az = fmaf(uz[j], h[j], az);
    ar = fmaf(ur[j], h[j], ar);
    ac = fmaf(uc[j], h[j], ac);
  }
  const float z = sigm(pz + az);
  const float r = sigm(pr + ar);
  const float c = tanh_f(fmaf(r, ac, pc));
  const float hi = h[i];  // h is in shared memory: a lane-dependent index is fine
  const float f = fmaf(z, c - hi, hi);
  const float da = (c - hi) * z * (1.0f - z);
  const float q = z * fmaf(-c, c, 1.0f);
  const float db = q * r;
  const float dc = q * ac * r * (1.0f - r);
  const float dz = 1.0f - z;
#pragma unroll
  for (int j = 0; j < 8; ++j)
    Jrow[j] = fmaf(da, uz[j], fmaf(db, uc[j], dc * ur[j])) + (j == i ? dz : 0.0f);
  return f;
}

template <typename PT>
__device__ __forceinline__ void mh2_stage(const MhParams& p, const PT* P, long long b, int g,
                                          long long D, long long t0, int k, Mh2Smem<PT>& sm,
                                          long long r, long long st, long long n) {
  // h^k of positions t0 .. t0 + T - 1 into rows 1..T (zeros at k = 0 and past n)
  for (int e = threadIdx.x; e < kMh2T * 2; e += kMh2Threads) {
    const int s = e >> 1, half = e & 1;
    const long long t = t0 + s;
    const bool valid = k > 0 && t < n;
    const float* src = valid ? p.h + (b * p.L + r + t * st) * D + 8 * g + 4 * half : p.h;
    cp_async16(smem_u32(sm.hk + mh2_hk(s) + 4 * half), src, valid);
  }
  constexpr int per = 24 * (int)sizeof(PT) / 16;  // 16-byte pieces per step (6 or 3)
  for (int e = threadIdx.x; e < kMh2T * per; e += kMh2Threads) {
    const int s = e / per, q = e - per * s;
    const long long t = t0 + s;
    const bool valid = t < n;
    const int first = q * 16 / (int)sizeof(PT);
    const PT* src =
        valid ? P + ((b * p.L + r + t * st) * 3 + first / 8) * D + 8 * g + (first % 8) : P;
    cp_async16(smem_u32(sm.gates + mh2_gate(s) + first), src, valid);
  }
  cp_async_commit();
}

template <typename PT>
__global__ void __launch_bounds__(kMh2Threads)
    pararnn_mhgru2_kernel(const MhParams p) {
  extern __shared__ __align__(16) unsigned char s_raw[];
  Mh2Smem<PT>& sm = *reinterpret_cast<Mh2Smem<PT>*>(s_raw);

  const int tid = threadIdx.x, lane = tid & 31;
  const int grp = tid >> 3;          // segment of the chunk this lane's group owns
  const int i = lane & 7;            // row / column of the 8x8 blocks this lane owns
  const unsigned gmask = 0xffu << (lane & 24);  // the group's 8 lanes
  const long long D = 8 * p.H;
  const WaitCtx wctx{p.ctrl, p.status_dev, p.timeout_ns};
  const PT* P = static_cast<const PT*>(p.P);

  const bool strided = p.offs != nullptr;
  const long long per_row = strided ? (long long)p.offs[p.H] : p.H;
  const bool bad_strides = strided && p.offs[p.H + 1] != 0;
  const long long nunits = bad_strides ? 0 : p.B * per_row;

  int last = -1;
  bool stop = false;
  for (int k = 0; !stop; ++k) {
    const bool update = k < p.max_iters;
    float rmax = 0.0f;
    for (long long u = blockIdx.x; u < nunits; u += gridDim.x) {
      const long long b = u / per_row;
      const long long rem = u - b * per_row;
      int g = (int)rem;
      long long r = 0, st = 1, n = p.L;
      if (strided) {
        int lo = 0, hi = (int)p.H - 1;
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if ((long long)p.offs[mid] <= rem) lo = mid; else hi = mid - 1;
        }
        g = lo;
        st = (long long)p.offs[g + 1] - p.offs[g];
        r = rem - p.offs[g];
        n = (p.L - r + st - 1) / st;
      }
      __syncthreads();  // the previous unit is done with shared memory
      for (int e = tid; e < 192; e += kMh2Threads)
        (&sm.U[0][0][0])[e] = __ldg(p.U + ((long long)(e >> 6) * p.H + g) * 64 + (e & 63));
      if (tid < 8) {
        const float v = p.h0 ? __ldg(p.h0 + b * D + 8 * g + tid) : 0.0f;
        sm.xin[kMh2Seg][tid] = v;  // h^{k+1} entering the first chunk
        sm.hk[tid] = v;            // h^k before the first step
      }
      __syncthreads();
      float uz[8], ur[8], uc[8];  // this lane's rows of the head's blocks
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        uz[j] = sm.U[0][i][j];
        ur[j] = sm.U[1][i][j];
        uc[j] = sm.U[2][i][j];
      }
      const int nch = (int)((n + kMh2T - 1) / kMh2T);

      for (int ci = 0; ci < nch; ++ci) {
        const long long t0 = (long long)ci * kMh2T;
        // rows 1..T of hk and the gates; row 0 keeps h^k of the step before the chunk
        mh2_stage<PT>(p, P, b, g, D, t0, k, sm, r, st, n);
        cp_async_wait_all();
        __syncthreads();
        // h^k of the chunk's last step: row 0 of the next chunk (written back after
        // the chunk's last read of row 0, while the next staging fills rows 1..T)
        const float hnext = tid < 8 ? sm.hk[mh2_hk(kMh2T - 1) + tid] : 0.0f;

        // ---- A: the group's segment: residual rows, Jacobian rows, its map ---------
        const int s0 = grp * kMh2S;
        float acol[8];  // column i of the segment map
#pragma unroll
        for (int m = 0; m < 8; ++m) acol[m] = (m == i) ? 1.0f : 0.0f;
        float boff = 0.0f;  // component i of the segment map's offset
        for (int s = 0; s < kMh2S; ++s) {
          const long long t = t0 + s0 + s;
          if (t >= n) break;  // uniform over the group (one segment per group)
          const float* hp = sm.hk + mh2_hk(s0 + s - 1);
          const PT* pg = sm.gates + mh2_gate(s0 + s);
          float Jrow[8];
          const float f =
              mh2_row(hp, uz, ur, uc, to_f(pg[i]), to_f(pg[8 + i]), to_f(pg[16 + i]), i, Jrow);
          rmax = max_abs_nan(rmax, f - sm.hk[mh2_hk(s0 + s) + i]);
          if (!update) continue;
          float bt = f;
#pragma unroll
          for (int j = 0; j < 8; ++j) bt = fmaf(-Jrow[j], hp[j], bt);
          // the group's Jacobian rows meet in shared memory
          float4* jr = reinterpret_cast<float4*>(&sm.J[grp][8 * i]);
          jr[0] = make_float4(Jrow[0], Jrow[1], Jrow[2], Jrow[3]);
          jr[1] = make_float4(Jrow[4], Jrow[5], Jrow[6], Jrow[7]);
          __syncwarp(gmask);
          // column i: A[:, i] <- J A[:, i]; offset: b_i <- (J b)_i + bt_i
          float nc[8];
#pragma unroll
          for (int row = 0; row < 8; ++row) {
            const float4 j0 = reinterpret_cast<const float4*>(&sm.J[grp][8 * row])[0];
            const float4 j1 = reinterpret_cast<const float4*>(&sm.J[grp][8 * row])[1];
            float v = j0.x * acol[0];
            v = fmaf(j0.y, acol[1], v);
            v = fmaf(j0.z, acol[2], v);
            v = fmaf(j0.w, acol[3], v);
            v = fmaf(j1.x, acol[4], v);
            v = fmaf(j1.y, acol[5], v);
            v = fmaf(j1.z, acol[6], v);
            v = fmaf(j1.w, acol[7], v);
            nc[row] = v;
          }
          float nb = bt;
#pragma unroll
          for (int m = 0; m < 8; ++m)
            nb = fmaf(Jrow[m], __shfl_sync(gmask, boff, (lane & 24) | m), nb);
#pragma unroll
          for (int m = 0; m < 8; ++m) acol[m] = nc[m];
          boff = nb;
          __syncwarp(gmask);  // every lane has read this step's rows before the next
        }

        if (update) {
          // ---- B: carry the chunk's incoming state through the segment maps --------
#pragma unroll
          for (int m = 0; m < 8; ++m) sm.A[grp][i][m] = acol[m];  // column i
          sm.bv[grp][i] = boff;
          __syncthreads();
          if (tid < 8) {
            // group 0 walks the segments; lane i keeps component i of the state
            float xi = sm.xin[kMh2Seg][i];  // the state leaving the previous chunk
            for (int kseg = 0; kseg < kMh2Seg; ++kseg) {
              sm.xin[kseg][i] = xi;
              __syncwarp(0xffu);
              float y = sm.bv[kseg][i];
#pragma unroll
              for (int m = 0; m < 8; ++m) y = fmaf(sm.A[kseg][m][i], sm.xin[kseg][m], y);
              __syncwarp(0xffu);
              xi = y;
            }
            sm.xin[kMh2Seg][i] = xi;  // the state leaving this chunk
          }
          __syncthreads();

          // ---- C: apply the segment's steps from its incoming state --------------
          float x[8];
#pragma unroll
          for (int m = 0; m < 8; ++m) x[m] = sm.xin[grp][m];
          for (int s = 0; s < kMh2S; ++s) {
            const long long t = t0 + s0 + s;
            if (t >= n) break;
            const float* hp = sm.hk + mh2_hk(s0 + s - 1);
            const PT* pg = sm.gates + mh2_gate(s0 + s);
            float Jrow[8];
            const float f =
                mh2_row(hp, uz, ur, uc, to_f(pg[i]), to_f(pg[8 + i]), to_f(pg[16 + i]), i, Jrow);
            float y = f;
#pragma unroll
            for (int j = 0; j < 8; ++j) y = fmaf(Jrow[j], x[j] - hp[j], y);
            p.h[(b * p.L + r + t * st) * D + 8 * g + i] = y;
#pragma unroll
            for (int m = 0; m < 8; ++m) x[m] = __shfl_sync(gmask, y, (lane & 24) | m);
          }
        }
        __syncthreads();  // the chunk's rows and maps are no longer read
        if (tid < 8) sm.hk[tid] = hnext;
      }
    }

    // ---- the global residual of iteration k; every CTA takes the same decision ----
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float o = __shfl_xor_sync(0xffffffffu, rmax, off);
      rmax = max_abs_nan(rmax, o);
    }
    if (lane == 0) atomicMax(&p.rho_bits[k], __float_as_uint(rmax));
    if (!grid_barrier(wctx)) break;
    last = k;
    const float rho = __uint_as_float(ld_volatile(&p.rho_bits[k]));
    stop = !(rho <= 3.0e38f) || rho <= p.tol || k >= p.max_iters;
  }

  if (blockIdx.x == 0 && threadIdx.x == 0) {
    struct Info {
      int iterations, converged, status, updates, passes, reserved;
      float max_residual;
      float rho[128];
    };
    Info* info = reinterpret_cast<Info*>(p.info);
    __threadfence();
    unsigned status = ld_volatile(&p.ctrl->status);
    if (bad_strides) status = 1u;  // PARARNN_ERR_INVALID_ARGUMENT: a stride below 1
    int iters = last, conv = 0, nonfinite = 0;
    float maxres = 0.0f;
    for (int kk = 0; kk <= p.max_iters; ++kk) {
      const float rv = kk <= last ? __uint_as_float(ld_volatile(&p.rho_bits[kk])) : 0.0f;
      info->rho[kk] = rv;
    }
    if (last >= 0) {
      maxres = info->rho[last];
      if (!(maxres <= 3.0e38f)) nonfinite = 1;
      else if (maxres <= p.tol) conv = 1;
    }
    if (status == 0u && nonfinite) status = 5u;
    info->iterations = iters < 0 ? 0 : iters;
    info->converged = (status == 0u) ? conv : 0;
    info->status = (int)status;
    info->updates = last < 0 ? 0 : (last < p.max_iters ? last + 1 : p.max_iters);
    info->passes = last + 1;
    info->reserved = 0;
    info->max_residual = maxres;
  }
}

}  // namespace pararnn
