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
// The chunk's gates and h^k arrive by cp.async copies into one of two
// shared-memory buffers while the previous chunk is being processed.
//
// Time strides (DEER summary, caveats paragraph: heads with exponentially
// increasing strides, i.e. shorter effective sequences): head g may recur at
// stride s_g, h_t = f(h_{t - s_g}, P_t).  Such a head is s_g independent
// sequences t = r, r + s_g, r + 2 s_g, ... (r < s_g), each solved exactly like a
// stride-1 sequence; a work unit is then (batch row, head, residue r), and the
// unit's positions k = 0, 1, ... address time step r + k s_g in memory.
#pragma once

#include "pararnn_kernel.cuh"
#include "pararnn_walk.cuh"

// Steps per lane and sequences per CTA, measured on B200 at B=8, L=4096, 128
// heads: 6 x 4, one buffer: 2.65 ms; 4 x 4: 3.2 ms; 8 x 4: 3.8 ms; two buffers
// (3 x 4): 2.85 ms -- the second buffer costs more occupancy than it hides.
#ifndef PARARNN_MH_STEPS
#define PARARNN_MH_STEPS 6
#endif
#ifndef PARARNN_MH_WARPS
#define PARARNN_MH_WARPS 4
#endif
// 1: the next chunk's copies are in flight while this one is processed (two
// buffers per warp); 0: one buffer, filled at the start of each chunk.
#ifndef PARARNN_MH_ASYNC
#define PARARNN_MH_ASYNC 0
#endif

namespace pararnn {

constexpr int kMhS = PARARNN_MH_STEPS;      // steps per lane per chunk
constexpr int kMhWarps = PARARNN_MH_WARPS;  // sequences (warps) per CTA
constexpr int kMhT = 32 * kMhS;             // steps per chunk
constexpr int kMhBufs = PARARNN_MH_ASYNC ? 2 : 1;

// Staged rows are grouped by lane (a lane's S consecutive steps), with 16 bytes
// of padding after each lane's block.  Lanes read their own rows at the same
// time; without the pad the lane blocks would sit 48 (h^k) or 144 (gates) words
// apart, always on the same two banks (a 16-way conflict).  With it a 16-byte
// read by 8 lanes hits 8 different bank groups.
constexpr int kMhHkLane = kMhS * 8 + 4;          // floats per lane block of h^k rows
template <typename PT> __host__ __device__ constexpr int mh_gate_lane() {
  return kMhS * 24 + 16 / (int)sizeof(PT);      // elements per lane block of gate rows
}
constexpr int kMhHkFloats = 8 + 32 * kMhHkLane;  // + the step before the chunk (first 8)
// h^k row of chunk position t (-1 = the step before the chunk); gate row of t
__host__ __device__ constexpr int mh_hk(int t) {
  return t < 0 ? 0 : 8 + (t / kMhS) * kMhHkLane + (t % kMhS) * 8;
}
template <typename PT> __host__ __device__ constexpr int mh_gate(int t) {
  return (t / kMhS) * mh_gate_lane<PT>() + (t % kMhS) * 24;
}
static_assert((kMhHkFloats * 4) % 16 == 0 && (kMhHkLane * 4) % 16 == 0, "16-byte rows");

// Dynamic shared memory per warp: one or two buffers of (h^k rows, gates of the chunk).
template <typename PT> __host__ __device__ constexpr size_t mh_buf_bytes() {
  return (size_t)kMhHkFloats * 4 + (size_t)32 * mh_gate_lane<PT>() * sizeof(PT);
}

// 8 h^k values and 24 gate values of one step as 16-byte shared-memory reads.
__device__ __forceinline__ void mh_ld8(const float* src, float* v) {
  const float4 a = reinterpret_cast<const float4*>(src)[0];
  const float4 c = reinterpret_cast<const float4*>(src)[1];
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = c.x; v[5] = c.y; v[6] = c.z; v[7] = c.w;
}
__device__ __forceinline__ void mh_ld_gates(const float* src, float* v) {
#pragma unroll
  for (int q = 0; q < 6; ++q) {
    const float4 a = reinterpret_cast<const float4*>(src)[q];
    v[4 * q] = a.x; v[4 * q + 1] = a.y; v[4 * q + 2] = a.z; v[4 * q + 3] = a.w;
  }
}
__device__ __forceinline__ void mh_ld_gates(const __nv_bfloat16* src, float* v) {
#pragma unroll
  for (int q = 0; q < 3; ++q) {
    const uint4 a = reinterpret_cast<const uint4*>(src)[q];
    const unsigned w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      v[8 * q + 2 * e] = __uint_as_float(w[e] << 16);
      v[8 * q + 2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
    }
  }
}
template <typename PT> __host__ __device__ constexpr size_t mh_smem_bytes() {
  return (size_t)kMhWarps * kMhBufs * mh_buf_bytes<PT>();
}

struct MhParams {
  const int* offs;     // NULL (every stride 1) or [H + 2]: offs[g] = sum of the
                       // heads' strides (each capped at L) before head g,
                       // offs[H] = their total, offs[H + 1] = 1 if a stride was < 1
  const void* P;       // [B, L, 3, D] (z, r, c), fp32 or bf16; D = 8 H; 16-byte aligned
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

// Cell and Jacobian of one head at h (row-major J[i][j] = dh'_i / dh_j).  U is
// the head's blocks in shared memory (16-byte aligned rows); each row of the
// three blocks is read once, as float4, for both the product and the Jacobian.
__device__ __forceinline__ void mh_cell(const float* p, const float* U, const float* h, float* f,
                                        float (*J)[8]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float u[3][8];
#pragma unroll
    for (int gt = 0; gt < 3; ++gt) {
      const float4 a = reinterpret_cast<const float4*>(U + (gt * 8 + i) * 8)[0];
      const float4 c = reinterpret_cast<const float4*>(U + (gt * 8 + i) * 8)[1];
      u[gt][0] = a.x; u[gt][1] = a.y; u[gt][2] = a.z; u[gt][3] = a.w;
      u[gt][4] = c.x; u[gt][5] = c.y; u[gt][6] = c.z; u[gt][7] = c.w;
    }
    float uz = 0.0f, ur = 0.0f, uc = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      uz = fmaf(u[0][j], h[j], uz);
      ur = fmaf(u[1][j], h[j], ur);
      uc = fmaf(u[2][j], h[j], uc);
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
    for (int j = 0; j < 8; ++j) J[i][j] = fmaf(da, u[0][j], fmaf(db, u[2][j], dc * u[1][j]));
    J[i][i] += 1.0f - z;
  }
}

// Issue the copies of chunk t0 into one buffer: h^k of steps t0 .. t0 + T - 1
// into rows 1..T (zeros at k = 0, where h^0 = 0, and past L) and their gates.
// Positions t0 .. t0 + T - 1 of a unit whose sequence has n positions; position
// k is time step r + k st in memory (r = 0, st = 1 without strides).
template <typename PT>
__device__ __forceinline__ void mh_issue_chunk(const MhParams& p, const PT* P, long long b, int g,
                                               long long D, long long t0, int k, float* hkb,
                                               PT* spb, int lane, long long r, long long st,
                                               long long n) {
  for (int e = lane; e < kMhT * 2; e += 32) {
    const int s = e >> 1, half = e & 1;
    const long long t = t0 + s;
    const bool valid = k > 0 && t < n;
    const float* src = valid ? p.h + (b * p.L + r + t * st) * D + 8 * g + 4 * half : p.h;
    cp_async16(smem_u32(hkb + mh_hk(s) + 4 * half), src, valid);
  }
  constexpr int per = 24 * (int)sizeof(PT) / 16;  // 16-byte pieces per step (6 or 3)
  for (int e = lane; e < kMhT * per; e += 32) {
    const int s = e / per, q = e - per * s;
    const long long t = t0 + s;
    const bool valid = t < n;
    // piece q covers gate (q * 16 / sizeof(PT)) / 8, channels from (q * 16 / sizeof(PT)) % 8
    const int first = q * 16 / (int)sizeof(PT);
    const PT* src =
        valid ? P + ((b * p.L + r + t * st) * 3 + first / 8) * D + 8 * g + (first % 8) : P;
    cp_async16(smem_u32(spb + mh_gate<PT>(s) + first), src, valid);
  }
  cp_async_commit();
}

template <typename PT>
__global__ void __launch_bounds__(32 * kMhWarps, 1) pararnn_mhgru_kernel(const MhParams p) {
  __shared__ __align__(16) float s_U[kMhWarps][3 * 64];
  extern __shared__ __align__(16) unsigned char s_dyn[];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long D = 8 * p.H;
  // work units: (batch row, head) sequences, or (batch row, head, residue) with strides
  const bool strided = p.offs != nullptr;
  const long long per_row = strided ? (long long)p.offs[p.H] : p.H;
  const bool bad_strides = strided && p.offs[p.H + 1] != 0;
  const long long nunits = bad_strides ? 0 : p.B * per_row;
  const WaitCtx wctx{p.ctrl, p.status_dev, p.timeout_ns};
  const PT* P = static_cast<const PT*>(p.P);
  unsigned char* wbase = s_dyn + (size_t)warp * kMhBufs * mh_buf_bytes<PT>();
  // buffer j: h^k rows, then the gates
  auto hkbuf = [&](int j) { return reinterpret_cast<float*>(wbase + j * mh_buf_bytes<PT>()); };
  auto spbuf = [&](int j) {
    return reinterpret_cast<PT*>(wbase + j * mh_buf_bytes<PT>() + kMhHkFloats * 4);
  };
  int last = -1;  // last iteration whose global residual is complete
  bool stop = false;

  for (int k = 0; !stop; ++k) {
    const bool update = k < p.max_iters;
    float rmax = 0.0f;
    for (long long u = (long long)blockIdx.x * kMhWarps + warp; u < nunits;
         u += (long long)gridDim.x * kMhWarps) {
      const long long b = u / per_row;
      const long long rem = u - b * per_row;
      int g = (int)rem;
      long long r = 0, st = 1, n = p.L;
      if (strided) {  // the head whose residues hold rem: the last g with offs[g] <= rem
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
      for (int e = lane; e < 192; e += 32)
        s_U[warp][e] = __ldg(p.U + ((long long)(e >> 6) * p.H + g) * 64 + (e & 63));
      float x[8], hb[8];  // entering the chunk: h^{k+1} and h^k (h0 before the first)
#pragma unroll
      for (int i = 0; i < 8; ++i) x[i] = hb[i] = p.h0 ? __ldg(p.h0 + b * D + 8 * g + i) : 0.0f;
      const float* U = s_U[warp];
      const int nch = (int)((n + kMhT - 1) / kMhT);
      if (kMhBufs == 2)
        mh_issue_chunk<PT>(p, P, b, g, D, 0, k, hkbuf(0), spbuf(0), lane, r, st, n);

      for (int ci = 0; ci < nch; ++ci) {
        const long long t0 = (long long)ci * kMhT;
        const int cur = kMhBufs == 2 ? (ci & 1) : 0;
        float* hk = hkbuf(cur);
        const PT* sp = spbuf(cur);
        if (kMhBufs == 1)
          mh_issue_chunk<PT>(p, P, b, g, D, t0, k, hk, spbuf(0), lane, r, st, n);
        cp_async_wait_all();
        __syncwarp();
        if (lane < 8) hk[lane] = hb[lane];  // row 0: h^k of the step before the chunk
        __syncwarp();
        if (kMhBufs == 2 && ci + 1 < nch)
          mh_issue_chunk<PT>(p, P, b, g, D, t0 + kMhT, k, hkbuf(cur ^ 1), spbuf(cur ^ 1), lane,
                             r, st, n);

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
          if (t >= n) break;
          float hp[8], hc[8], pg[24], f[8], J[8][8];
          mh_ld8(hk + mh_hk(s0 + s - 1), hp);
          mh_ld8(hk + mh_hk(s0 + s), hc);
          mh_ld_gates(sp + mh_gate<PT>(s0 + s), pg);
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
          // (A, bv) <- (J A, J bv + bt), column by column
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
            if (t >= n) break;
            float hp[8], pg[24], f[8], J[8][8];
            mh_ld8(hk + mh_hk(s0 + s - 1), hp);
            mh_ld_gates(sp + mh_gate<PT>(s0 + s), pg);
            mh_cell(pg, U, hp, f, J);
            float y[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              float s2 = f[i];
#pragma unroll
              for (int j = 0; j < 8; ++j) s2 = fmaf(J[i][j], xin[j] - hp[j], s2);
              y[i] = s2;
            }
            float4* dst = reinterpret_cast<float4*>(p.h + (b * p.L + r + t * st) * D + 8 * g);
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
        for (int i = 0; i < 8; ++i) hb[i] = hk[mh_hk(kMhT - 1) + i];
        __syncwarp();  // the buffer is refilled by a later chunk
      }
      cp_async_wait_all();
      __syncwarp();  // s_U and the buffers are reused by the next sequence
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
    if (bad_strides) status = 1u;  // PARARNN_ERR_INVALID_ARGUMENT: a stride below 1
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
