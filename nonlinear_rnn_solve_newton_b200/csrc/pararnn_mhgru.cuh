// pararnn_mhgru.cuh -- Newton solve of the multi-head GRU whose recurrence is
// block-diagonal with dense 8x8 blocks (one block per head of 8 channels).
//
// The dense-block case the DEER summary's caveats price at O(n^3) per step
// (n = 8 here): per head the Newton step is a block bi-diagonal system with
// dense 8x8 Jacobians, solved by a scan of affine maps x -> A x + b.  Cell, per
// head (elementwise products):
//   z = sig(P_z + U_z h), r = sig(P_r + U_r h), c = tanh(P_c + r (U_c h)),
//   h' = (1 - z) h + z c,
//   J = diag(1 - z) + diag((c - h) z (1 - z)) U_z + diag(z (1 - c^2) r) U_c
//       + diag(z (1 - c^2) (U_c h) r (1 - r)) U_r,
// i.e. the ParaGRU cell when every block is diagonal.
//
// Organisation: one warp per (batch row, head) sequence, walking time chunks
// of 32 lanes x S steps; CTAs are persistent (cooperative launch) and iterate
// Newton in place, with a grid barrier and the global max-abs residual between
// iterations (the same stopping rule as the diagonal solves).  Per chunk:
//   A. each lane linearises its S steps at h^k (cell, 8x8 Jacobian, residual)
//      and composes their maps into one segment map (8x8 matrix kept by
//      columns, so composing needs no second matrix);
//   B. the state entering each lane's segment is handed from lane to lane
//      (one 8x8 matrix-vector product per lane, a serial chain over 32 lanes);
//   C. each lane recomputes its steps' maps and applies them from that state,
//      writing h^{k+1} over h^k (the chunk's h^k was staged in shared memory
//      first, so no lane reads an overwritten value).
// The chunk's gate inputs are staged in shared memory too, by coalesced loads
// that are all in flight at once, so neither phase waits on global memory.
#pragma once

#include "pararnn_kernel.cuh"

// Steps per lane and sequences per CTA, measured on B200 at B=8, L=4096,
// 128 heads (4 x 4 with staged gates: 4.1 ms; 8-16 steps: 4.8 ms; 32: 8.4 ms).
#ifndef PARARNN_MH_STEPS
#define PARARNN_MH_STEPS 4
#endif
#ifndef PARARNN_MH_WARPS
#define PARARNN_MH_WARPS 4
#endif
#ifndef PARARNN_MH_STAGE_P
#define PARARNN_MH_STAGE_P 1
#endif

namespace pararnn {

constexpr int kMhS = PARARNN_MH_STEPS;  // steps per lane per chunk
constexpr int kMhWarps = PARARNN_MH_WARPS;  // sequences (warps) per CTA
constexpr int kMhT = 32 * kMhS;             // steps per chunk
// dynamic shared memory per warp: h^k of the chunk ((T + 1) x 8) and its gates (T x 24)
constexpr bool kMhStageP = PARARNN_MH_STAGE_P != 0;
constexpr size_t kMhWarpFloats = (size_t)(kMhT + 1) * 8 + (kMhStageP ? (size_t)kMhT * 24 : 0);
constexpr size_t kMhSmem = (size_t)kMhWarps * kMhWarpFloats * sizeof(float);

struct MhParams {
  const void* P;       // [B, L, 3, D] (z, r, c), fp32 or bf16; D = 8 H
  const float* U;      // [3, H, 8, 8]: gate, head, row (output), column (input)
  const float* h0;     // [B, D] or NULL (= 0)
  float* h;            // [B, L, D]: the iterate, updated in place; the result
  long long B, L, H;
  float tol;
  int max_iters;
  Ctrl* ctrl;
  unsigned* rho_bits;  // [max_iters + 1], max-abs residual per iteration (float bits)
  void* info;          // pararnn_solve_info_t (device)
  int* status_dev;
  long long timeout_ns;
};

// Cell and Jacobian of one head at h (row-major J[i][j] = dh'_i / dh_j).
__device__ __forceinline__ void mh_cell(const float* p, const float (*U)[8][8], const float* h,
                                        float* f, float (*J)[8]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float uz = 0.0f, ur = 0.0f, uc = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      uz = fmaf(U[0][i][j], h[j], uz);
      ur = fmaf(U[1][i][j], h[j], ur);
      uc = fmaf(U[2][i][j], h[j], uc);
    }
    const float z = sigm(p[i] + uz);
    const float r = sigm(p[8 + i] + ur);
    const float c = tanh_f(fmaf(r, uc, p[16 + i]));
    f[i] = fmaf(z, c - h[i], h[i]);
    const float da = (c - h[i]) * z * (1.0f - z);
    const float q = z * fmaf(-c, c, 1.0f);
    const float db = q * r;
    const float dc = q * uc * r * (1.0f - r);
#pragma unroll
    for (int j = 0; j < 8; ++j)
      J[i][j] = fmaf(da, U[0][i][j], fmaf(db, U[2][i][j], dc * U[1][i][j]));
    J[i][i] += 1.0f - z;
  }
}

template <typename PT>
__device__ __forceinline__ void mh_load_gates(const PT* P, long long row, long long D, int g,
                                              float* p) {
  const PT* q = P + row * 3 * D + 8 * g;
#pragma unroll
  for (int k = 0; k < 3; ++k)
#pragma unroll
    for (int i = 0; i < 8; ++i) p[8 * k + i] = to_f(__ldg(q + k * D + i));
}

// Stage the gates of steps t0 .. t0 + T - 1 of head g, batch row b into
// sp[s][24] (z, r, c x 8 channels); steps past L are zero.
template <typename PT>
__device__ __forceinline__ void mh_stage_gates(const PT* P, long long b, long long t0, long long L,
                                               long long D, int g, float* sp, int lane) {
  if constexpr (sizeof(PT) == 4) {
    // 6 float4 per step (3 gates x 8 channels)
    for (int e = lane; e < kMhT * 6; e += 32) {
      const int s = e / 6, q = e - 6 * s;  // q: gate = q / 2, half = q % 2
      const long long t = t0 + s;
      float4 v = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      if (t < L)
        v = __ldg(reinterpret_cast<const float4*>(P + ((b * L + t) * 3 + (q >> 1)) * D + 8 * g) +
                  (q & 1));
      reinterpret_cast<float4*>(sp)[e] = v;
    }
  } else {
    // 3 x 16 bytes (8 bf16) per step
    for (int e = lane; e < kMhT * 3; e += 32) {
      const int s = e / 3, gate = e - 3 * s;
      const long long t = t0 + s;
      float f[8];
      if (t < L) {
        const uint4 v =
            __ldg(reinterpret_cast<const uint4*>(P + ((b * L + t) * 3 + gate) * D + 8 * g));
        const unsigned w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          f[2 * i] = __uint_as_float(w[i] << 16);
          f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) f[i] = 0.0f;
      }
      float4* d = reinterpret_cast<float4*>(sp + 24 * s + 8 * gate);
      d[0] = make_float4(f[0], f[1], f[2], f[3]);
      d[1] = make_float4(f[4], f[5], f[6], f[7]);
    }
  }
}

template <typename PT>
__global__ void __launch_bounds__(32 * kMhWarps, 1) pararnn_mhgru_kernel(const MhParams p) {
  __shared__ float s_U[kMhWarps][3][8][8];
  // per warp, h^k of the chunk: row 0 = the step before it, row s + 1 = step s
  extern __shared__ float s_hk[];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long D = 8 * p.H;
  const long long nunits = p.B * p.H;
  const WaitCtx wctx{p.ctrl, p.status_dev, p.timeout_ns};
  const PT* P = static_cast<const PT*>(p.P);  // 16-byte aligned rows of 8 channels
  int last = -1;  // last iteration whose global residual is complete
  bool stop = false;

  for (int k = 0; !stop; ++k) {
    const bool update = k < p.max_iters;
    float rmax = 0.0f;
    for (long long u = (long long)blockIdx.x * kMhWarps + warp; u < nunits;
         u += (long long)gridDim.x * kMhWarps) {
      const long long b = u / p.H;
      const int g = (int)(u - b * p.H);
      for (int e = lane; e < 192; e += 32)
        (&s_U[warp][0][0][0])[e] = __ldg(p.U + ((long long)(e >> 6) * p.H + g) * 64 + (e & 63));
      float x[8], hb[8];  // state entering the chunk: h^{k+1} and h^k
#pragma unroll
      for (int i = 0; i < 8; ++i) x[i] = hb[i] = p.h0 ? __ldg(p.h0 + b * D + 8 * g + i) : 0.0f;
      __syncwarp();
      const float(*U)[8][8] = s_U[warp];
      float* hk = s_hk + (size_t)warp * kMhWarpFloats;
      float* sp = hk + (kMhT + 1) * 8;

      for (long long t0 = 0; t0 < p.L; t0 += kMhT) {
        // ---- stage h^k of the chunk (zero at k = 0: h^0 = 0) --------------------
        if (lane < 8) hk[lane] = hb[lane];
        for (int e = lane; e < kMhT * 8; e += 32) {
          const long long t = t0 + (e >> 3);
          hk[8 + e] = (k > 0 && t < p.L) ? p.h[(b * p.L + t) * D + 8 * g + (e & 7)] : 0.0f;
        }
        if constexpr (kMhStageP) mh_stage_gates<PT>(P, b, t0, p.L, D, g, sp, lane);
        __syncwarp();

        // ---- A: linearise this lane's steps, compose their maps ------------------
        const int s0 = lane * kMhS;
        float A[8][8], bv[8];  // segment map, A[j][i] = column j, row i
#pragma unroll
        for (int j = 0; j < 8; ++j) {
#pragma unroll
          for (int i = 0; i < 8; ++i) A[j][i] = (i == j) ? 1.0f : 0.0f;
          bv[j] = 0.0f;
        }
        for (int s = 0; s < kMhS; ++s) {
          const long long t = t0 + s0 + s;
          if (t >= p.L) break;
          float hp[8], hc[8], f[8], J[8][8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            hp[i] = hk[(s0 + s) * 8 + i];
            hc[i] = hk[(s0 + s + 1) * 8 + i];
          }
          float pg[24];
          if constexpr (kMhStageP) {
#pragma unroll
            for (int i = 0; i < 24; ++i) pg[i] = sp[24 * (s0 + s) + i];
          } else {
            mh_load_gates<PT>(P, b * p.L + t, D, g, pg);
          }
          mh_cell(pg, U, hp, f, J);
          float bt[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            rmax = max_abs_nan(rmax, f[i] - hc[i]);
            float s2 = f[i];
#pragma unroll
            for (int j = 0; j < 8; ++j) s2 = fmaf(-J[i][j], hp[j], s2);
            bt[i] = s2;
          }
          // (A, bv) <- (J A, J bv + bt)
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            float col[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              float s2 = 0.0f;
#pragma unroll
              for (int m = 0; m < 8; ++m) s2 = fmaf(J[i][m], A[j][m], s2);
              col[i] = s2;
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) A[j][i] = col[i];
          }
          float nb[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            float s2 = bt[i];
#pragma unroll
            for (int m = 0; m < 8; ++m) s2 = fmaf(J[i][m], bv[m], s2);
            nb[i] = s2;
          }
#pragma unroll
          for (int i = 0; i < 8; ++i) bv[i] = nb[i];
        }

        if (update) {
          // ---- B: the state entering each lane's segment, lane to lane ----------
          float xin[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) xin[i] = x[i];
          for (int j = 0; j < 31; ++j) {
            float y[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              float s2 = bv[i];
#pragma unroll
              for (int m = 0; m < 8; ++m) s2 = fmaf(A[m][i], xin[m], s2);
              y[i] = s2;
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float v = __shfl_sync(0xffffffffu, y[i], j);
              if (lane == j + 1) xin[i] = v;
            }
          }

          // ---- C: recompute and apply this lane's steps, write h^{k+1} ----------
          for (int s = 0; s < kMhS; ++s) {
            const long long t = t0 + s0 + s;
            if (t >= p.L) break;
            float hp[8], f[8], J[8][8];
#pragma unroll
            for (int i = 0; i < 8; ++i) hp[i] = hk[(s0 + s) * 8 + i];
            float pg[24];
            if constexpr (kMhStageP) {
#pragma unroll
              for (int i = 0; i < 24; ++i) pg[i] = sp[24 * (s0 + s) + i];
            } else {
              mh_load_gates<PT>(P, b * p.L + t, D, g, pg);
            }
            mh_cell(pg, U, hp, f, J);
            float y[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              float s2 = f[i];
#pragma unroll
              for (int j = 0; j < 8; ++j) s2 = fmaf(J[i][j], xin[j] - hp[j], s2);
              y[i] = s2;
            }
            float4* dst = reinterpret_cast<float4*>(p.h + (b * p.L + t) * D + 8 * g);
            dst[0] = make_float4(y[0], y[1], y[2], y[3]);
            dst[1] = make_float4(y[4], y[5], y[6], y[7]);
#pragma unroll
            for (int i = 0; i < 8; ++i) xin[i] = y[i];
          }
          // state leaving the chunk: the last lane's (full chunks only continue)
#pragma unroll
          for (int i = 0; i < 8; ++i) x[i] = __shfl_sync(0xffffffffu, xin[i], 31);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) hb[i] = hk[kMhT * 8 + i];
        __syncwarp();  // s_hk is restaged by the next chunk
      }
      __syncwarp();  // s_U is reloaded by the next sequence
    }

    // ---- global residual of iteration k, then every CTA takes the same decision
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
    int iters = last, conv = 0, nonfinite = 0;
    float maxres = 0.0f;
    for (int kk = 0; kk <= p.max_iters; ++kk) {
      const float r = kk <= last ? __uint_as_float(ld_volatile(&p.rho_bits[kk])) : 0.0f;
      info->rho[kk] = r;
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
