// pararnn_walk.cuh -- the tile-walking kernel: one CTA per tile of 32 channels,
// time chunks staged in shared memory by TMA, all iterations of a sweep on chip.
//
// Same method and arithmetic as pararnn_kernel (ParaRNN TL;DR / Abstract: Newton
// on the stacked system, each step a bi-diagonal solve by a parallel
// reduction), organised for the case where the channel tiles alone fill the
// GPU (LM-width layers):
//   * the CTA walks the chunks of its tile in time order; the state entering
//     chunk j at iteration k (h^{k+1} at the chunk start, and h^k for the
//     Jacobian) is what chunk j-1 produced at the same iteration, kept in
//     shared memory -- no traffic between CTAs at all;
//   * the projected inputs of chunk j+1 are fetched by one TMA tensor copy
//     (cp.async.bulk.tensor, box = 32 channels x gates x T steps) into the other
//     half of a double buffer while chunk j is being iterated, so registers hold
//     only the iterate and the step maps;
//   * one __syncthreads per Newton iteration: every warp composes the
//     aggregates of the warps before it (double-buffered shared array) and
//     applies them to the carry it already has.
#pragma once

#include <cuda.h>

#include "pararnn_kernel.cuh"

namespace pararnn {

struct TmaMaps {
  CUtensorMap in0;  // P (solves) or A (scans)
  CUtensorMap in1;  // b (scans)
};

__device__ __forceinline__ unsigned smem_u32(const void* p) {
  return static_cast<unsigned>(__cvta_generic_to_shared(p));
}

// 16-byte asynchronous copy global -> shared; with valid == false it writes
// zeros and reads nothing.  Copies are committed in groups and waited for by
// group, oldest first.
__device__ __forceinline__ void cp_async16(unsigned dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_group 0;" ::: "memory");
}
// all but the most recently committed group have landed
__device__ __forceinline__ void cp_async_wait_prior() {
  asm volatile("cp.async.wait_group 1;" ::: "memory");
}
__device__ __forceinline__ void mbar_init(unsigned long long* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(unsigned long long* bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(unsigned long long* bar, unsigned parity) {
  unsigned ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0u;
}
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y,
                                            unsigned long long* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<unsigned long long>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int x, int y, int z,
                                            unsigned long long* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<unsigned long long>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}

// Shared-memory image of one time chunk, per op: [T][G][CW] for CW channels.
template <int OP, typename PT, int TCH, int CW = 32> struct Stage;
template <typename PT, int TCH, int CW> struct Stage<kGru, PT, TCH, CW> {
  static constexpr unsigned kBytes = TCH * 3 * CW * sizeof(PT);
  __device__ static void issue(unsigned char* s, const TmaMaps& tm, int d0, int row,
                               unsigned long long* bar) {
    mbar_expect_tx(bar, kBytes);
    tma_load_3d(s, &tm.in0, d0, 0, row, bar);
  }
  __device__ static void read(const unsigned char* s, int tl, int c, float* v) {
    const PT* q = reinterpret_cast<const PT*>(s) + tl * 3 * CW + c;
    v[0] = to_f(q[0]);
    v[1] = to_f(q[CW]);
    v[2] = to_f(q[2 * CW]);
  }
};
// 8-channel LSTM tiles: one plane per gate, [G][T][8] (four tensor copies of
// 8 channels x 1 gate x T rows).  Rows of 8 channels put a warp's four time
// segments on different shared-memory banks when the steps per segment are
// odd; one [T][G][8] image would give rows of 32 words, a 4-way conflict.
template <typename PT, int TCH> struct Stage<kLstm, PT, TCH, 8> {
  static constexpr unsigned kPlane = TCH * 8 * sizeof(PT);
  static_assert(kPlane % 128 == 0, "gate planes stay 128-byte aligned");
  static constexpr unsigned kBytes = 4 * kPlane;
  __device__ static void issue(unsigned char* s, const TmaMaps& tm, int d0, int row,
                               unsigned long long* bar) {
    mbar_expect_tx(bar, kBytes);
#pragma unroll
    for (int g = 0; g < 4; ++g) tma_load_3d(s + g * kPlane, &tm.in0, d0, g, row, bar);
  }
  __device__ static void read(const unsigned char* s, int tl, int c, float* v) {
    const PT* q = reinterpret_cast<const PT*>(s) + tl * 8 + c;
#pragma unroll
    for (int g = 0; g < 4; ++g) v[g] = to_f(q[g * (TCH * 8)]);
  }
};
template <typename PT, int TCH, int CW> struct Stage<kLstm, PT, TCH, CW> {
  static constexpr unsigned kBytes = TCH * 4 * CW * sizeof(PT);
  __device__ static void issue(unsigned char* s, const TmaMaps& tm, int d0, int row,
                               unsigned long long* bar) {
    mbar_expect_tx(bar, kBytes);
    tma_load_3d(s, &tm.in0, d0, 0, row, bar);
  }
  __device__ static void read(const unsigned char* s, int tl, int c, float* v) {
    const PT* q = reinterpret_cast<const PT*>(s) + tl * 4 * CW + c;
    v[0] = to_f(q[0]);
    v[1] = to_f(q[CW]);
    v[2] = to_f(q[2 * CW]);
    v[3] = to_f(q[3 * CW]);
  }
};
template <typename PT, int TCH, int CW> struct Stage<kScanDiag, PT, TCH, CW> {
  static constexpr unsigned kHalf = TCH * CW * 4;
  static constexpr unsigned kBytes = 2 * kHalf;
  __device__ static void issue(unsigned char* s, const TmaMaps& tm, int d0, int row,
                               unsigned long long* bar) {
    mbar_expect_tx(bar, kBytes);
    tma_load_2d(s, &tm.in0, d0, row, bar);
    tma_load_2d(s + kHalf, &tm.in1, d0, row, bar);
  }
  __device__ static void read(const unsigned char* s, int tl, int c, float* v) {
    v[0] = reinterpret_cast<const float*>(s)[tl * CW + c];
    v[1] = reinterpret_cast<const float*>(s + kHalf)[tl * CW + c];
  }
};
template <typename PT, int TCH, int CW> struct Stage<kScanBlock2, PT, TCH, CW> {
  static_assert(CW == 32, "the 2x2 scan walker stages 32-channel tiles");
  static constexpr unsigned kA = TCH * 32 * 16;
  static constexpr unsigned kBytes = kA + TCH * 32 * 8;
  __device__ static void issue(unsigned char* s, const TmaMaps& tm, int d0, int row,
                               unsigned long long* bar) {
    mbar_expect_tx(bar, kBytes);
    tma_load_2d(s, &tm.in0, 4 * d0, row, bar);
    tma_load_2d(s + kA, &tm.in1, 2 * d0, row, bar);
  }
  __device__ static void read(const unsigned char* s, int tl, int c, float* v) {
    const float4 a = reinterpret_cast<const float4*>(s)[tl * 32 + c];
    const float2 b = reinterpret_cast<const float2*>(s + kA)[tl * 32 + c];
    v[0] = a.x;
    v[1] = a.y;
    v[2] = a.z;
    v[3] = a.w;
    v[4] = b.x;
    v[5] = b.y;
  }
};

// Bounded wait for a stage's bytes to land.
__device__ __forceinline__ bool stage_wait(unsigned long long* bar, unsigned parity,
                                           const WaitCtx& w) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer();
  for (;;) {
    if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer() - t0 > (unsigned long long)w.timeout_ns) return false;
  }
}

// Before a CTA exits: wait for the copies still in flight into its shared
// memory (thread 0; bit s of `pending` = stage s, `phase` = the parities).  The
// copies read valid global memory and land within microseconds; the limit is at
// least 2 s so that a short user wait limit, which may have ended a stage wait
// early, cannot let the CTA leave before its copies do.
__device__ __forceinline__ void drain_stages(unsigned long long* bars, unsigned pending,
                                             unsigned phase, const WaitCtx& w) {
  WaitCtx wl = w;
  if (wl.timeout_ns < 2000000000LL) wl.timeout_ns = 2000000000LL;
  for (int st = 0; st < 2; ++st)
    if (pending & (1u << st)) stage_wait(&bars[st], (phase >> st) & 1u, wl);
}

template <int OP, typename PT, int S, int NW, int MINB, int CW = 32>
__global__ void __launch_bounds__(NW * 32, MINB)
    pararnn_walk_kernel(const __grid_constant__ KParams p, const __grid_constant__ TmaMaps tm) {
  using T_ = OpT<OP>;
  constexpr int NS = T_::NS;
  constexpr int NI = T_::NI;
  constexpr bool NEWTON = T_::newton;
  static_assert(CW == 32 || CW == 16 || CW == 8, "tile width");
  constexpr int SPL = 32 / CW;       // segments per warp (lane = channel + CW * segment)
  constexpr int NSEG = NW * SPL;     // segments per chunk, S steps each
  constexpr int TCH = NSEG * S;      // steps per chunk
  using St = Stage<OP, PT, TCH, CW>;
  constexpr unsigned kStageBytes = (St::kBytes + 1023u) / 1024u * 1024u;
  constexpr int WM = kMaxWalkIters;

  extern __shared__ __align__(1024) unsigned char dsmem[];
  __shared__ unsigned long long s_bar[2];
  __shared__ Map<NS> s_wagg[2][NW][CW];   // per-segment aggregates, double-buffered by iteration
  __shared__ Vec<NS> s_inc[2][WM][CW];    // chunk-end state per iteration, by chunk parity
  __shared__ Vec<NS> s_pend[2][CW];       // chunk-end state of the loaded iterate
  __shared__ unsigned s_racc[WM];
  __shared__ int s_item;
  __shared__ int s_flag;

  const WaitCtx wctx{p.ctrl, p.status_dev, p.timeout_ns};
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int c = lane % CW;        // channel within the tile
  const int sub = lane / CW;      // segment within the warp
  const int seg = warp * SPL + sub;
  const bool last_in_warp = sub == SPL - 1;

  if (tid == 0) {
    mbar_init(&s_bar[0], 1);
    mbar_init(&s_bar[1], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  __syncthreads();

  unsigned phase = 0u;    // parity of the next wait, per stage (bit s)
  unsigned pending = 0u;  // stages with a copy in flight (thread 0's view)
  int k0 = 0;
  int q = 0;
  bool aborted = false;

  for (;; ++q) {
    const int m = NEWTON ? sweep_len(q, k0, p.m_first, p.m_next, p.max_iters) : 1;

    // The first tile of a sweep is the CTA's own (blockIdx.x < ntiles: the grid
    // is never larger than the tile count); later ones are drawn from a counter.
    for (int first = 1;; first = 0) {  // tiles
      if (tid == 0) {
        int u = p.ntiles;
        if (first) {
          u = (int)blockIdx.x;
        } else if ((int)gridDim.x < p.ntiles) {
          u = (int)gridDim.x + (int)atomicAdd(&p.ticket[q], 1u);
          if (ld_volatile(&p.ctrl->abort) != 0u) u = p.ntiles;
        }
        s_item = u;
      }
      if (tid < WM) s_racc[tid] = 0u;
      __syncthreads();
      const int tile = s_item;
      if (tile >= p.ntiles) break;

      const long long b = tile / p.ntd;
      const int td = tile - (int)b * p.ntd;
      const int d0 = td * CW;
      const long long d = d0 + c;
      const bool cvalid = d < p.D;
      const long long bd = b * p.D + d;
      const int row0 = (int)(b * p.L);

      float wv[NEWTON ? NI : 1];
      Vec<NS> x0v;
#pragma unroll
      for (int i = 0; i < NS; ++i) x0v.x[i] = 0.0f;
      if (cvalid) IO<OP, PT>::init_state(p, bd, x0v.x);
      if constexpr (NEWTON) {
#pragma unroll
        for (int g = 0; g < NI; ++g) wv[g] = cvalid ? __ldg(p.w + (long long)g * p.D + d) : 0.0f;
      }

      // first two chunks of the tile in flight
      if (tid == 0) {
        for (int jj = 0; jj < 2 && jj < p.nchunks; ++jj) {
          St::issue(dsmem + jj * kStageBytes, tm, d0, row0 + jj * TCH, &s_bar[jj]);
          pending |= 1u << jj;
        }
      }

      for (int j = 0; j < p.nchunks; ++j) {
        const int st = j & 1;
        const unsigned char* stage = dsmem + st * kStageBytes;
        const long long t0 = (long long)j * TCH + (long long)seg * S;
        const bool full = cvalid && (t0 + S) <= p.L;

        // ---- current iterate and the state before this segment -----------
        Vec<NS> x[S];
        Vec<NS> xb;
#pragma unroll
        for (int i = 0; i < NS; ++i) xb.x[i] = 0.0f;
        if constexpr (NEWTON) {
          if (k0 == 0) {
#pragma unroll
            for (int s = 0; s < S; ++s)
#pragma unroll
              for (int i = 0; i < NS; ++i) x[s].x[i] = 0.0f;
            if (t0 == 0) xb = x0v;
          } else {
#pragma unroll
            for (int s = 0; s < S; ++s) {
              const long long t = t0 + s;
              if (cvalid && t < p.L) {
                IO<OP, PT>::load_state(p, (b * p.L + t) * p.D + d, x[s].x);
              } else {
#pragma unroll
                for (int i = 0; i < NS; ++i) x[s].x[i] = 0.0f;
              }
            }
            if (t0 == 0) {
              xb = x0v;
            } else if (seg == 0) {
              xb = s_pend[(j - 1) & 1][c];
            } else if (cvalid && t0 - 1 < p.L) {
              IO<OP, PT>::load_state(p, (b * p.L + t0 - 1) * p.D + d, xb.x);
            }
            if (seg == NSEG - 1) s_pend[j & 1][c] = x[S - 1];
          }
        }

        // ---- this chunk's inputs have landed ------------------------------
        const bool ok = stage_wait(&s_bar[st], (phase >> st) & 1u, wctx);
        if (ok) {  // a copy that did not land stays pending for the final drain
          phase ^= 1u << st;
          if (tid == 0) pending &= ~(1u << st);
        }
        if (!__syncthreads_and(ok ? 1 : 0)) {
          if (tid == 0) raise_error(wctx, 4u);
          aborted = true;
          break;
        }

        bool any_update = false;
        for (int kk = 0; kk < m; ++kk) {
          const int k = k0 + kk;
          const bool upd = !NEWTON || k < p.max_iters;

          Map<NS> mp[S];
          Map<NS> agg = map_identity<NS>();
          float rmax = 0.0f;
          Vec<NS> xp = xb;
          if (full) {
#pragma unroll
            for (int s = 0; s < S; ++s) {
              float vin[NI];
              St::read(stage, seg * S + s, c, vin);
              if constexpr (NEWTON) {
                mp[s] = newton_step<OP>(vin, wv, xp, x[s], rmax);
                xp = x[s];
              } else {
                mp[s] = StepMap<OP>::from_inputs(vin);
              }
              agg = compose(mp[s], agg);
            }
          } else {
#pragma unroll
            for (int s = 0; s < S; ++s) {
              if (cvalid && (t0 + s) < p.L) {
                float vin[NI];
                St::read(stage, seg * S + s, c, vin);
                if constexpr (NEWTON) {
                  mp[s] = newton_step<OP>(vin, wv, xp, x[s], rmax);
                  xp = x[s];
                } else {
                  mp[s] = StepMap<OP>::from_inputs(vin);
                }
              } else {
                mp[s] = map_identity<NS>();
              }
              agg = compose(mp[s], agg);
            }
          }
          if constexpr (NEWTON) {
            const unsigned rbits = __reduce_max_sync(0xffffffffu, __float_as_uint(rmax));
            if (lane == 0) atomicMax(&s_racc[kk], rbits);
          }
          if (!upd) continue;  // residual-only iteration (k == max_iters)
          any_update = true;

          // ---- combine the segments: one barrier per iteration ---------------
          // Each warp composes the aggregates of the warps before it (the shared
          // array alternates between iterations, so the next iteration's writes
          // cannot overtake a slow warp's reads) and applies the prefix to the
          // state carried in from the previous chunk at this iteration.
          const int buf = kk & 1;
          // segments of this warp: inclusive scan over the lanes of each channel
          Map<NS> wincl = agg, wexcl = map_identity<NS>();
          if constexpr (SPL > 1) {
#pragma unroll
            for (int off = CW; off < 32; off <<= 1) {
              const Map<NS> o = shfl_up_map(wincl, off);
              if (lane >= off) wincl = compose(wincl, o);
            }
            const Map<NS> e = shfl_up_map(wincl, CW);
            if (sub > 0) wexcl = e;
          }
          if (last_in_warp) s_wagg[buf][warp][c] = wincl;
          __syncthreads();
          Map<NS> pre = map_identity<NS>();
#pragma unroll 4
          for (int w2 = 0; w2 < warp; ++w2) pre = compose(s_wagg[buf][w2][c], pre);
          const Vec<NS> carry = (j == 0) ? x0v : s_inc[(j - 1) & 1][kk][c];
          const Vec<NS> xin = apply(wexcl, apply(pre, carry));
          if (warp == NW - 1 && last_in_warp) s_inc[j & 1][kk][c] = apply(agg, xin);
          Vec<NS> xr = xin;
#pragma unroll
          for (int s = 0; s < S; ++s) {
            xr = apply(mp[s], xr);
            x[s] = xr;
          }
          xb = xin;
        }

        // ---- write the chunk; refill its stage with chunk j + 2 -----------
        if (any_update || k0 == 0 || !NEWTON) {
          if (full) {
#pragma unroll
            for (int s = 0; s < S; ++s)
              IO<OP, PT>::store_state(p, (b * p.L + t0 + s) * p.D + d, x[s].x);
          } else {
#pragma unroll
            for (int s = 0; s < S; ++s) {
              const long long t = t0 + s;
              if (cvalid && t < p.L) IO<OP, PT>::store_state(p, (b * p.L + t) * p.D + d, x[s].x);
            }
          }
        }
        __syncthreads();  // every warp is done reading this stage
        if (tid == 0 && j + 2 < p.nchunks) {
          St::issue(dsmem + st * kStageBytes, tm, d0, row0 + (j + 2) * TCH, &s_bar[st]);
          pending |= 1u << st;
        }
      }
      if (aborted) break;
      if constexpr (NEWTON) {
        if (tid < m) atomicMax(&p.rho_bits[k0 + tid], s_racc[tid]);
      }
      __syncthreads();
    }
    if (aborted) break;

    if constexpr (!NEWTON) {
      break;
    } else {
      if (!grid_barrier(wctx)) {
        aborted = true;
        break;
      }
      // The stop rule and the report below are written out here rather than
      // through sweep_stops / write_solve_info: with the helpers the LM-width
      // walker measured 1-2 % slower on B200 (same registers; the hot loop is
      // sensitive to how the kernel's tail compiles).
      if (tid == 0) {
        int done = 0;
        for (int kk = 0; kk < m; ++kk) {
          const float r = __uint_as_float(ld_volatile(&p.rho_bits[k0 + kk]));
          if (!(r <= 3.0e38f)) {
            done = 1;
            break;
          }
          if (r <= p.tol) done = 1;
        }
        if (k0 + m > p.max_iters) done = 1;
        s_flag = done;
      }
      __syncthreads();
      if (s_flag) break;
      k0 += m;
    }
  }

  // No copy may still be writing this CTA's shared memory when it exits.
  if (tid == 0 && pending) drain_stages(s_bar, pending, phase, wctx);

  if constexpr (NEWTON) {
    if (blockIdx.x == 0 && tid == 0) {
      struct Info {
        int iterations, converged, status, updates, passes, reserved;
        float max_residual;
        float rho[128];
      };
      Info* info = reinterpret_cast<Info*>(p.info);
      __threadfence();
      unsigned status = ld_volatile(&p.ctrl->status);
      const int last = k0 + sweep_len(q, k0, p.m_first, p.m_next, p.max_iters) - 1;
      int iters = p.max_iters, conv = 0, nonfinite = 0;
      float maxres = 0.0f;
      for (int k = 0; k <= last && k <= p.max_iters; ++k) {
        const float r = __uint_as_float(ld_volatile(&p.rho_bits[k]));
        info->rho[k] = r;
        if (!(r <= 3.0e38f)) nonfinite = 1;
      }
      for (int k = 0; k <= last && k <= p.max_iters; ++k) {
        const float r = __uint_as_float(ld_volatile(&p.rho_bits[k]));
        iters = k;
        maxres = r;
        if (!(r <= 3.0e38f)) break;
        if (r <= p.tol) {
          conv = 1;
          break;
        }
      }
      for (int k = last + 1; k <= p.max_iters; ++k) info->rho[k] = 0.0f;
      if (status == 0u && nonfinite) status = 5u;
      info->iterations = iters;
      info->converged = (status == 0u) ? conv : 0;
      info->status = (int)status;
      info->updates = last < p.max_iters ? last + 1 : p.max_iters;
      info->passes = q + 1;
      info->reserved = 0;
      info->max_residual = maxres;
    }
  }
}

}  // namespace pararnn
