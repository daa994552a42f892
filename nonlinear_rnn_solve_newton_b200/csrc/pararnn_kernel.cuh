// pararnn_kernel.cuh -- the sm_100a kernel behind libpararnn.so.
//
// One persistent kernel template serves the four operations of the ParaRNN /
// DEER hot path ("ParaRNN: Unlocking Parallel Training of Nonlinear RNNs for
// Large Language Models", TL;DR, Abstract and Figure 2; DEER summary):
//
//   * the diagonal and 2x2 affine scans  x_t = A_t x_{t-1} + b_t  (the linear
//     solve of a Newton step: a block bi-diagonal system), and
//   * the ParaGRU / ParaLSTM Newton solves of h_t = f(h_{t-1}, P_t), where each
//     iteration evaluates the cell, its (block-)diagonal Jacobian and the
//     residual at every step and then solves the bi-diagonal system.
//
// Work decomposition.  The trajectory [B, L, D] is cut into units of
// (CW consecutive channels along D) x (T consecutive steps).  Inside a
// 256-thread CTA, thread (seg, c) owns channel c of the tile and the S steps
// [t0 + seg*S, t0 + (seg+1)*S) of the chunk, with NSEG = 256 / CW segments and
// T = NSEG * S.  Units are handed out by an atomic ticket in chunk-major
// order, so every predecessor of a unit (the same tile, earlier chunks) was
// handed out first and is already running: the look-back below always makes
// progress.
//
// One Newton iteration inside a unit (all in registers / shared memory):
//   1. per step, at the current iterate: f, A = df/dh, the residual
//      r = f - h^k_t (its max goes to an atomic per iteration), and the affine
//      map  h^{k+1}_t = A h^{k+1}_{t-1} + (f - A h^k_{t-1});
//   2. each thread composes its S maps serially;
//   3. warp shuffles compose the segments inside a warp, shared memory the 8
//      warps, giving the unit's aggregate map per channel;
//   4. decoupled look-back along the chunk chain of the tile: publish the
//      aggregate, walk back over predecessors' aggregates until an inclusive
//      value, publish the inclusive value (the new state at the chunk end);
//   5. apply the carried-in state through the maps: h^{k+1} for the S steps.
// The inputs P stay in registers across the m iterations of a sweep, so a
// sweep reads P once and h once and writes h once whatever m is.  Sweeps are
// separated by a grid barrier (the kernel is launched cooperatively, all CTAs
// resident), after which every CTA reads the per-iteration residual maxima and
// takes the same stop decision: Newton's stopping rule on the global max, as
// in the Figure 4 caption.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

namespace pararnn {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

enum OpKind : int { kScanDiag = 0, kScanBlock2 = 1, kGru = 2, kLstm = 3 };

// NS: state components per channel (1 diagonal, 2 block).  NI: input values per
// step held in registers.
template <int OP> struct OpT;
template <> struct OpT<kScanDiag> {
  static constexpr int NS = 1, NI = 2;
  static constexpr bool newton = false;
};
template <> struct OpT<kScanBlock2> {
  static constexpr int NS = 2, NI = 6;
  static constexpr bool newton = false;
};
template <> struct OpT<kGru> {
  static constexpr int NS = 1, NI = 3;
  static constexpr bool newton = true;
};
template <> struct OpT<kLstm> {
  static constexpr int NS = 2, NI = 4;
  static constexpr bool newton = true;
};

// ---------------------------------------------------------------------------
// Workspace control block (zeroed by the host before each launch).
// ---------------------------------------------------------------------------
struct Ctrl {
  unsigned bar_count;  // grid-barrier arrivals (only grows: (g + 1) x grid after barrier g)
  unsigned bar_gen;    // grid barriers completed
  unsigned abort;
  unsigned status;
  unsigned pad[12];
  // followed by: unsigned rho_bits[max_iters + 1]; unsigned ticket[npasses]
};

struct KParams {
  const void* in0;       // P (solves) or A (scans)
  const float* in1;      // b (scans)
  const float* w;        // recurrence weights [G, D] (solves)
  const float* x0a;      // h0 (GRU, diag scan), c0 (LSTM), x0 (block scan)
  const float* x0b;      // h0 (LSTM)
  float* out0;           // h (GRU, diag scan), c (LSTM), x (block scan)
  float* out1;           // h (LSTM)
  long long B, L, D;
  int ntd;               // tiles along D
  int ntiles;            // B * ntd
  int nchunks;
  int nunits;
  float tol;
  int max_iters;
  int m_first, m_next, mmax;
  Ctrl* ctrl;
  unsigned* rho_bits;    // [max_iters + 1]
  unsigned* ticket;      // [npasses]
  unsigned long long* rec;  // look-back records [mmax][nunits][CW][Rec<NS>::kWords]
  float* bnd;            // [2][nunits][CW][NS]
  int vec1;              // D == 1 and every array 16-byte aligned with L % 8 == 0:
                         // a thread's S steps are one contiguous, aligned block
  void* info;            // pararnn_solve_info_t* (solves)
  int* status_dev;       // scans, optional
  long long timeout_ns;
  long long stall_unit;
};

// ---------------------------------------------------------------------------
// Memory-model helpers (PTX acquire/release at GPU scope, L2-coherent loads).
// ---------------------------------------------------------------------------
__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release(unsigned* p, unsigned v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ unsigned ld_volatile(const unsigned* p) {
  return *reinterpret_cast<const volatile unsigned*>(p);
}
__device__ __forceinline__ unsigned long long globaltimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ float ldcg(const float* p) { return __ldcg(p); }

// ---------------------------------------------------------------------------
// Affine maps x -> M x + v and their composition.
// ---------------------------------------------------------------------------
template <int NS> struct Map {
  float m[NS][NS];
  float v[NS];
};

template <int NS> __device__ __forceinline__ Map<NS> map_identity() {
  Map<NS> r;
#pragma unroll
  for (int i = 0; i < NS; ++i) {
#pragma unroll
    for (int j = 0; j < NS; ++j) r.m[i][j] = (i == j) ? 1.0f : 0.0f;
    r.v[i] = 0.0f;
  }
  return r;
}

// later o earlier: x -> later(earlier(x))
template <int NS>
__device__ __forceinline__ Map<NS> compose(const Map<NS>& later, const Map<NS>& earlier) {
  Map<NS> r;
#pragma unroll
  for (int i = 0; i < NS; ++i) {
#pragma unroll
    for (int j = 0; j < NS; ++j) {
      float s = later.m[i][0] * earlier.m[0][j];
#pragma unroll
      for (int k = 1; k < NS; ++k) s = fmaf(later.m[i][k], earlier.m[k][j], s);
      r.m[i][j] = s;
    }
    float s = later.v[i];
#pragma unroll
    for (int k = 0; k < NS; ++k) s = fmaf(later.m[i][k], earlier.v[k], s);
    r.v[i] = s;
  }
  return r;
}

template <int NS> struct Vec {
  float x[NS];
};

template <int NS>
__device__ __forceinline__ Vec<NS> apply(const Map<NS>& M, const Vec<NS>& x) {
  Vec<NS> y;
#pragma unroll
  for (int i = 0; i < NS; ++i) {
    float s = M.v[i];
#pragma unroll
    for (int k = 0; k < NS; ++k) s = fmaf(M.m[i][k], x.x[k], s);
    y.x[i] = s;
  }
  return y;
}

template <int NS>
__device__ __forceinline__ Map<NS> shfl_up_map(const Map<NS>& a, int delta) {
  Map<NS> r;
#pragma unroll
  for (int i = 0; i < NS; ++i) {
#pragma unroll
    for (int j = 0; j < NS; ++j) r.m[i][j] = __shfl_up_sync(0xffffffffu, a.m[i][j], delta);
    r.v[i] = __shfl_up_sync(0xffffffffu, a.v[i], delta);
  }
  return r;
}

// Shuffle up within independent groups of `width` lanes.
template <int NS>
__device__ __forceinline__ Map<NS> shfl_up_map_w(const Map<NS>& a, int delta, int width) {
  Map<NS> r;
#pragma unroll
  for (int i = 0; i < NS; ++i) {
#pragma unroll
    for (int j = 0; j < NS; ++j) r.m[i][j] = __shfl_up_sync(0xffffffffu, a.m[i][j], delta, width);
    r.v[i] = __shfl_up_sync(0xffffffffu, a.v[i], delta, width);
  }
  return r;
}

// ---------------------------------------------------------------------------
// Look-back records.  Every published number travels in its own aligned 64-bit
// word together with the sweep's tag (high 32 bits = tag, low 32 = the float).
// An aligned 64-bit access is single-copy atomic, so a reader validates each
// word by its tag alone: the writer needs no fence and the reader no separate
// flag round trip.  Per (iteration slot, unit, channel) the record holds the
// chunk aggregate (NS*NS matrix entries, then NS offsets) and the chunk-end
// state (NS words).  The records are zeroed before every call; tag 0 = empty.
// ---------------------------------------------------------------------------
template <int NS> struct Rec {
  static constexpr int kAgg = NS * NS + NS;
  static constexpr int kWords = kAgg + NS;
};

__device__ __forceinline__ unsigned long long tagged(unsigned tag, float v) {
  return ((unsigned long long)tag << 32) | (unsigned long long)__float_as_uint(v);
}
__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_relaxed_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

template <int NS>
__device__ __forceinline__ void publish_agg(unsigned long long* rec, unsigned tag,
                                            const Map<NS>& a) {
#pragma unroll
  for (int i = 0; i < NS; ++i)
#pragma unroll
    for (int j = 0; j < NS; ++j) st_relaxed_u64(rec + i * NS + j, tagged(tag, a.m[i][j]));
#pragma unroll
  for (int i = 0; i < NS; ++i) st_relaxed_u64(rec + NS * NS + i, tagged(tag, a.v[i]));
}
template <int NS>
__device__ __forceinline__ void publish_inc(unsigned long long* rec, unsigned tag,
                                            const Vec<NS>& x) {
#pragma unroll
  for (int i = 0; i < NS; ++i) st_relaxed_u64(rec + Rec<NS>::kAgg + i, tagged(tag, x.x[i]));
}

// ---------------------------------------------------------------------------
// Cells.  From the identities e^x = 2^(x log2 e),
//   sigma(x) = 1 / (1 + 2^(-x log2 e)),   tanh(x) = 1 - 2 / (1 + 2^(2 x log2 e)),
// each evaluated with one hardware base-2 exponential and one hardware
// reciprocal (PTX ex2.approx / rcp.approx: relative errors near 2^-22, so the
// per-step absolute error stays ~1e-7, far inside the 1e-4 parity bound).
// The limits are exact: 2^(+inf) = inf gives 1/inf = 0, 2^(-inf) = 0 gives 1.
// tanh.approx is not used: its ~2^-11 relative error would bias every step.
// ---------------------------------------------------------------------------
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float sigm(float x) {
  return rcp_approx(1.0f + ex2_approx(-kLog2e * x));
}
__device__ __forceinline__ float tanh_f(float x) {
  return fmaf(-2.0f, rcp_approx(1.0f + ex2_approx((2.0f * kLog2e) * x)), 1.0f);
}
// max(m, |r|) that keeps a NaN (PTX max.NaN): a NaN residual must stop the solve.
__device__ __forceinline__ float max_abs_nan(float m, float r) {
  float y;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(y) : "f"(m), "f"(fabsf(r)));
  return y;
}

// s (1 - s), the logistic derivative, as s - s^2 in one fused multiply-add
// (measured on B200: 1-2% off the GRU and LSTM solves against s * (1 - s)).
__device__ __forceinline__ float dsig(float s) { return fmaf(-s, s, s); }

// ParaGRU: h' = (1-z) h + z c; returns f and dh'/dh.
__device__ __forceinline__ void gru_cell(const float* p, const float* w, float h, float& f,
                                         float& J) {
  float z = sigm(fmaf(w[0], h, p[0]));
  float r = sigm(fmaf(w[1], h, p[1]));
  float rh = r * h;
  float c = tanh_f(fmaf(w[2], rh, p[2]));
  float cmh = c - h;
  f = fmaf(z, cmh, h);
  float dz = dsig(z) * w[0];
  float dr = dsig(r) * w[1];
  float du = w[2] * fmaf(h, dr, r);
  float dc = fmaf(-c, c, 1.0f) * du;
  J = fmaf(cmh, dz, 1.0f - z) + z * dc;
}

// ParaLSTM: state (c, h); f = (c', h'), J = d(c',h')/d(c,h) row-major.
__device__ __forceinline__ void lstm_cell(const float* p, const float* w, float c, float h,
                                          float& fc, float& fh, float J[2][2]) {
  float ig = sigm(fmaf(w[0], h, p[0]));
  float fg = sigm(fmaf(w[1], h, p[1]));
  float gg = tanh_f(fmaf(w[2], h, p[2]));
  float og = sigm(fmaf(w[3], h, p[3]));
  float cn = fmaf(fg, c, ig * gg);
  float tc = tanh_f(cn);
  fc = cn;
  fh = og * tc;
  float di = dsig(ig) * w[0];
  float df = dsig(fg) * w[1];
  float dg = fmaf(-gg, gg, 1.0f) * w[2];
  float dov = dsig(og) * w[3];
  float dcn_dh = fmaf(df, c, fmaf(di, gg, ig * dg));
  float odtc = og * fmaf(-tc, tc, 1.0f);
  J[0][0] = fg;
  J[0][1] = dcn_dh;
  J[1][0] = odtc * fg;
  J[1][1] = fmaf(dov, tc, odtc * dcn_dh);
}

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

// Residual maxima travel as the bits of a non-negative float: for those the
// unsigned order is the float order, and a NaN (0x7fc00000 or above) sorts
// above +Inf, so integer max reductions and atomics keep it visible.

// ---------------------------------------------------------------------------
// Bounded waits.
// ---------------------------------------------------------------------------
// What a bounded wait needs: where to raise an error, and the bound.
struct WaitCtx {
  Ctrl* ctrl;
  int* status_dev;
  long long timeout_ns;
};

__device__ __forceinline__ void raise_error(const WaitCtx& w, unsigned code) {
  atomicCAS(&w.ctrl->status, 0u, code);
  if (w.status_dev) atomicCAS(w.status_dev, 0, (int)code);
  __threadfence();
  atomicExch(&w.ctrl->abort, 1u);
}

// One non-blocking read of a look-back record by this lane: 2 = chunk-end state
// valid (in `inc`), 1 = aggregate valid (in `agg`), 0 = not yet published.
template <int NS>
__device__ __forceinline__ unsigned poll_record(const unsigned long long* rec, unsigned tag,
                                                Map<NS>& agg, Vec<NS>& inc) {
  unsigned long long q[Rec<NS>::kWords];
#pragma unroll
  for (int i = 0; i < Rec<NS>::kWords; ++i) q[i] = ld_relaxed_u64(rec + i);
  bool iok = true, aok = true;
#pragma unroll
  for (int i = 0; i < Rec<NS>::kAgg; ++i) aok = aok && (unsigned)(q[i] >> 32) == tag;
#pragma unroll
  for (int i = 0; i < NS; ++i) {
    iok = iok && (unsigned)(q[Rec<NS>::kAgg + i] >> 32) == tag;
    inc.x[i] = __uint_as_float((unsigned)q[Rec<NS>::kAgg + i]);
  }
#pragma unroll
  for (int i = 0; i < NS; ++i)
#pragma unroll
    for (int j = 0; j < NS; ++j) agg.m[i][j] = __uint_as_float((unsigned)q[i * NS + j]);
#pragma unroll
  for (int i = 0; i < NS; ++i) agg.v[i] = __uint_as_float((unsigned)q[NS * NS + i]);
  return iok ? 2u : (aok ? 1u : 0u);
}

template <int NS>
__device__ __forceinline__ Map<NS> shfl_down_map(const Map<NS>& a, int delta) {
  Map<NS> r;
#pragma unroll
  for (int i = 0; i < NS; ++i) {
#pragma unroll
    for (int j = 0; j < NS; ++j) r.m[i][j] = __shfl_down_sync(0xffffffffu, a.m[i][j], delta);
    r.v[i] = __shfl_down_sync(0xffffffffu, a.v[i], delta);
  }
  return r;
}
template <int NS>
__device__ __forceinline__ Vec<NS> shfl_vec(const Vec<NS>& a, int src) {
  Vec<NS> r;
#pragma unroll
  for (int i = 0; i < NS; ++i) r.x[i] = __shfl_sync(0xffffffffu, a.x[i], src);
  return r;
}

// Windowed look-back (all 32 lanes of one warp).  Lane (w, c) = (lane / CW,
// lane % CW) reads the record of predecessor w (counting back from the nearest,
// `first_pred`) for channel c, so one round trip covers WIN = min(32 / CW, 4)
// predecessors (a wider window measured slower: the nearest record is usually
// ready, and polling more of them costs more than the round trips it saves).  Per channel: the nearest predecessor holding a chunk-end state
// is found; the aggregates in front of it are composed by a shuffle tree
// (nearest = latest map first) and applied to that state.  A window of
// aggregates only is folded into `acc` and the window moves back; a window with
// an unpublished slot in front of the nearest state is re-read.  Returns false
// on timeout or abort; on success lanes < CW hold their channel's carry.
#ifndef PARARNN_LOOKBACK_WINDOW
#define PARARNN_LOOKBACK_WINDOW 4
#endif
template <int NS, int CW>
__device__ __forceinline__ bool window_lookback(const unsigned long long* rec_base,
                                                size_t unit_words, int first_pred, int unit_step,
                                                unsigned tag, Vec<NS>& carry, const WaitCtx& wc) {
  constexpr int WIN_MAX = 32 / CW;
  constexpr int WIN = WIN_MAX < PARARNN_LOOKBACK_WINDOW ? WIN_MAX : PARARNN_LOOKBACK_WINDOW;
  constexpr int RW = Rec<NS>::kWords;
  const int lane = threadIdx.x & 31;
  const int c = lane % CW;
  const int wi = lane / CW;
  Map<NS> acc = map_identity<NS>();  // windows already folded in, nearest first
  bool done = false;
  int base = first_pred;
  unsigned long long t_start = 0;
  bool timing = false;
  unsigned ns = 32;
  for (;;) {
    const int pu = base - wi * unit_step;
    Map<NS> agg = map_identity<NS>();
    Vec<NS> inc;
#pragma unroll
    for (int i = 0; i < NS; ++i) inc.x[i] = 0.0f;
    unsigned st = 0u;
    if (wi < WIN && pu >= 0 && !done)
      st = poll_record<NS>(rec_base + (size_t)pu * unit_words + (size_t)c * RW, tag, agg, inc);
    const unsigned inc_mask = __ballot_sync(0xffffffffu, st == 2u);
    const unsigned rdy_mask = __ballot_sync(0xffffffffu, st != 0u);
    int fw = WIN;
    bool gap = false;
#pragma unroll 1
    for (int w = 0; w < WIN; ++w) {
      const unsigned bit = 1u << (w * CW + c);
      if (inc_mask & bit) {
        fw = w;
        break;
      }
      if (!(rdy_mask & bit)) {
        gap = true;
        break;
      }
    }
    if (done) gap = false;
    if (!__any_sync(0xffffffffu, gap)) {
      Map<NS> m = (wi < fw) ? agg : map_identity<NS>();
#pragma unroll
      for (int off = CW; off < CW * WIN; off <<= 1) {
        const Map<NS> o = shfl_down_map(m, off);
        if (wi + off / CW < WIN) m = compose(m, o);
      }
      const Vec<NS> v = shfl_vec(inc, (fw < WIN ? fw : 0) * CW + c);
      if (!done) {
        acc = compose(acc, m);
        if (fw < WIN) {
          carry = apply(acc, v);
          done = true;
        }
      }
      if (__all_sync(0xffffffffu, done || wi != 0)) return true;
      base -= WIN * unit_step;
      continue;
    }
    if (!timing) {
      t_start = globaltimer();
      timing = true;
    }
    const bool aborting = __any_sync(0xffffffffu, ld_volatile(&wc.ctrl->abort) != 0u);
    const bool expired =
        __any_sync(0xffffffffu, (globaltimer() - t_start) > (unsigned long long)wc.timeout_ns);
    if (aborting || expired) {
      if (lane == 0 && !aborting) raise_error(wc, 4u /*TIMEOUT*/);
      return false;
    }
    __nanosleep(ns);
    if (ns < 256) ns <<= 1;
  }
}

// Global stop rule after a sweep of m iterations from k0: stop at the first
// iterate whose residual is within tol, on a non-finite residual, or once the
// iteration limit is reached.  The m loads are independent.
__device__ __forceinline__ int sweep_stops(const unsigned* rho_bits, int k0, int m, int max_iters,
                                           float tol) {
  int done = k0 + m > max_iters ? 1 : 0;
  for (int kk = 0; kk < m; ++kk) {
    const float r = __uint_as_float(ld_volatile(&rho_bits[k0 + kk]));
    if (!(r <= 3.0e38f) || r <= tol) done = 1;
  }
  return done;
}

// Grid-wide barrier (all CTAs are co-resident: cooperative launch).  The
// arrival counter only grows: every CTA arrives once per barrier and none can
// arrive at the next one before this one completes, so an arrival's count tells
// which barrier it belongs to (count / gridDim.x) and the last arrival of
// barrier g releases it by publishing g + 1.  Nothing is read before arriving
// and nothing is reset, so a barrier costs one atomic round trip plus the
// release.  Bounded; returns false if the kernel is aborting or the wait ran
// out.  The signature stays one small struct: the callers' hot loops compile as
// if the call were not there.
__device__ __noinline__ bool grid_barrier(WaitCtx p) {
  __shared__ int s_ok;
  __threadfence();  // every thread: its iterate and residuals before the CTA arrives
  __syncthreads();
  if (threadIdx.x == 0) {
    int ok = 1;
    const unsigned arrived = atomicAdd(&p.ctrl->bar_count, 1u);
    const unsigned next = arrived / gridDim.x + 1u;
    if (arrived == next * gridDim.x - 1u) {
      st_release(&p.ctrl->bar_gen, next);
    } else {
      const unsigned long long t0 = globaltimer();
      unsigned ns = 32;
      while (ld_acquire(&p.ctrl->bar_gen) < next) {
        if (ld_volatile(&p.ctrl->abort) != 0u) {
          ok = 0;
          break;
        }
        if (globaltimer() - t0 > (unsigned long long)p.timeout_ns) {
          raise_error(p, 4u);
          ok = 0;
          break;
        }
        __nanosleep(ns);
        if (ns < 256) ns <<= 1;
      }
    }
    s_ok = ok;
  }
  __syncthreads();
  return s_ok != 0;
}

// The solve's report (pararnn_solve_info_t), written by one thread once every
// CTA has finished: residuals rho_0..rho_last (zero after), the iteration count
// (the first iterate within tol, or the first non-finite residual, else the
// last evaluated), convergence and status.  `extra_status` replaces a zero
// status (e.g. a wait that ran out in this thread's own CTA).
__device__ __noinline__ void write_solve_info(void* info_ptr, Ctrl* ctrl,
                                                 const unsigned* rho_bits, int last, int passes,
                                                 int max_iters, float tol, unsigned extra_status) {
  struct Info {
    int iterations, converged, status, updates, passes, reserved;
    float max_residual;
    float rho[128];
  };
  Info* info = reinterpret_cast<Info*>(info_ptr);
  __threadfence();
  unsigned status = ld_volatile(&ctrl->status);
  if (status == 0u) status = extra_status;
  int iters = max_iters, conv = 0, nonfinite = 0;
  bool found = false;
  float maxres = 0.0f;
  for (int k = 0; k <= max_iters; ++k) {
    const float r = k <= last ? __uint_as_float(ld_volatile(&rho_bits[k])) : 0.0f;
    info->rho[k] = r;
    if (k > last) continue;
    const bool bad = !(r <= 3.0e38f);
    if (bad) nonfinite = 1;
    if (!found) {
      iters = k;
      maxres = r;
      if (bad) {
        found = true;
      } else if (r <= tol) {
        conv = 1;
        found = true;
      }
    }
  }
  if (status == 0u && nonfinite) status = 5u;
  info->iterations = iters;
  info->converged = (status == 0u) ? conv : 0;
  info->status = (int)status;
  info->updates = last < max_iters ? last + 1 : max_iters;
  info->passes = passes;
  info->reserved = 0;
  info->max_residual = maxres;
}

// Iterations evaluated in sweep q that starts at iteration k0.
__device__ __host__ __forceinline__ int sweep_len(int q, int k0, int m_first, int m_next,
                                                  int max_iters) {
  int m = (q == 0) ? m_first : m_next;
  int left = max_iters + 1 - k0;
  return m < left ? m : left;
}

// ---------------------------------------------------------------------------
// Per-op input and state access.
// ---------------------------------------------------------------------------
template <int OP, typename PT> struct IO;

template <typename PT> struct IO<kGru, PT> {
  __device__ static void load_in(const KParams& p, long long idx_btd, long long b, long long t,
                                 long long d, float* v) {
    const PT* P = reinterpret_cast<const PT*>(p.in0);
    long long base = ((b * p.L + t) * 3) * p.D + d;
#pragma unroll
    for (int g = 0; g < 3; ++g) v[g] = to_f(__ldg(P + base + g * p.D));
  }
  __device__ static void load_state(const KParams& p, long long i, float* x) {
    x[0] = ldcg(p.out0 + i);
  }
  __device__ static void store_state(const KParams& p, long long i, const float* x) {
    p.out0[i] = x[0];
  }
  __device__ static void init_state(const KParams& p, long long bd, float* x) {
    x[0] = p.x0a ? p.x0a[bd] : 0.0f;
  }
};

template <typename PT> struct IO<kLstm, PT> {
  __device__ static void load_in(const KParams& p, long long idx_btd, long long b, long long t,
                                 long long d, float* v) {
    const PT* P = reinterpret_cast<const PT*>(p.in0);
    long long base = ((b * p.L + t) * 4) * p.D + d;
#pragma unroll
    for (int g = 0; g < 4; ++g) v[g] = to_f(__ldg(P + base + g * p.D));
  }
  __device__ static void load_state(const KParams& p, long long i, float* x) {
    x[0] = ldcg(p.out0 + i);
    x[1] = ldcg(p.out1 + i);
  }
  __device__ static void store_state(const KParams& p, long long i, const float* x) {
    p.out0[i] = x[0];
    p.out1[i] = x[1];
  }
  __device__ static void init_state(const KParams& p, long long bd, float* x) {
    x[0] = p.x0a ? p.x0a[bd] : 0.0f;
    x[1] = p.x0b ? p.x0b[bd] : 0.0f;
  }
};

template <typename PT> struct IO<kScanDiag, PT> {
  __device__ static void load_in(const KParams& p, long long i, long long, long long, long long,
                                 float* v) {
    v[0] = __ldg(reinterpret_cast<const float*>(p.in0) + i);
    v[1] = __ldg(p.in1 + i);
  }
  __device__ static void load_state(const KParams& p, long long i, float* x) {
    x[0] = ldcg(p.out0 + i);
  }
  __device__ static void store_state(const KParams& p, long long i, const float* x) {
    p.out0[i] = x[0];
  }
  __device__ static void init_state(const KParams& p, long long bd, float* x) {
    x[0] = p.x0a ? p.x0a[bd] : 0.0f;
  }
};

template <typename PT> struct IO<kScanBlock2, PT> {
  __device__ static void load_in(const KParams& p, long long i, long long, long long, long long,
                                 float* v) {
    float4 a = __ldg(reinterpret_cast<const float4*>(p.in0) + i);
    float2 b = __ldg(reinterpret_cast<const float2*>(p.in1) + i);
    v[0] = a.x;
    v[1] = a.y;
    v[2] = a.z;
    v[3] = a.w;
    v[4] = b.x;
    v[5] = b.y;
  }
  __device__ static void load_state(const KParams& p, long long i, float* x) {
    float2 q = __ldcg(reinterpret_cast<const float2*>(p.out0) + i);
    x[0] = q.x;
    x[1] = q.y;
  }
  __device__ static void store_state(const KParams& p, long long i, const float* x) {
    reinterpret_cast<float2*>(p.out0)[i] = make_float2(x[0], x[1]);
  }
  __device__ static void init_state(const KParams& p, long long bd, float* x) {
    if (p.x0a) {
      float2 q = reinterpret_cast<const float2*>(p.x0a)[bd];
      x[0] = q.x;
      x[1] = q.y;
    } else {
      x[0] = 0.0f;
      x[1] = 0.0f;
    }
  }
};

// ---------------------------------------------------------------------------
// D == 1: a thread's S consecutive steps of one channel are one contiguous
// block of memory; move it with 16-byte vector accesses (the host checks the
// alignment and sets p.vec1).
// ---------------------------------------------------------------------------
template <typename T, int N>
__device__ __forceinline__ void ld_block(const T* src, float* dst) {
  constexpr int V = 16 / (int)sizeof(T);
  static_assert((N * (int)sizeof(T)) % 16 == 0, "block must be whole 16-byte vectors");
#pragma unroll
  for (int i = 0; i < N / V; ++i) {
    const uint4 q = __ldg(reinterpret_cast<const uint4*>(src) + i);
    T tmp[V];
    memcpy(tmp, &q, 16);
#pragma unroll
    for (int k = 0; k < V; ++k) dst[i * V + k] = to_f(tmp[k]);
  }
}
template <int N>
__device__ __forceinline__ void ld_block_cg(const float* src, float* dst) {
  static_assert(N % 4 == 0, "block must be whole float4s");
#pragma unroll
  for (int i = 0; i < N / 4; ++i) {
    const float4 q = __ldcg(reinterpret_cast<const float4*>(src) + i);
    dst[4 * i] = q.x;
    dst[4 * i + 1] = q.y;
    dst[4 * i + 2] = q.z;
    dst[4 * i + 3] = q.w;
  }
}
template <int N>
__device__ __forceinline__ void st_block(float* dst, const float* src) {
  static_assert(N % 4 == 0, "block must be whole float4s");
#pragma unroll
  for (int i = 0; i < N / 4; ++i)
    reinterpret_cast<float4*>(dst)[i] =
        make_float4(src[4 * i], src[4 * i + 1], src[4 * i + 2], src[4 * i + 3]);
}

// Per op: inputs of S steps [t0, t0+S) of channel b (D == 1) into vin[s][i], and
// the state block into / out of x[s].
template <int OP, typename PT, int S> struct Block1;
template <typename PT, int S> struct Block1<kGru, PT, S> {
  __device__ static void load_in(const KParams& p, long long b, long long t0, float (*vin)[3]) {
    ld_block<PT, 3 * S>(reinterpret_cast<const PT*>(p.in0) + (b * p.L + t0) * 3, &vin[0][0]);
  }
  __device__ static void load_state(const KParams& p, long long i0, Vec<1>* x) {
    float t[S];
    ld_block_cg<S>(p.out0 + i0, t);
#pragma unroll
    for (int s = 0; s < S; ++s) x[s].x[0] = t[s];
  }
  __device__ static void store_state(const KParams& p, long long i0, const Vec<1>* x) {
    float t[S];
#pragma unroll
    for (int s = 0; s < S; ++s) t[s] = x[s].x[0];
    st_block<S>(p.out0 + i0, t);
  }
};
template <typename PT, int S> struct Block1<kLstm, PT, S> {
  __device__ static void load_in(const KParams& p, long long b, long long t0, float (*vin)[4]) {
    ld_block<PT, 4 * S>(reinterpret_cast<const PT*>(p.in0) + (b * p.L + t0) * 4, &vin[0][0]);
  }
  __device__ static void load_state(const KParams& p, long long i0, Vec<2>* x) {
    float tc[S], th[S];
    ld_block_cg<S>(p.out0 + i0, tc);
    ld_block_cg<S>(p.out1 + i0, th);
#pragma unroll
    for (int s = 0; s < S; ++s) {
      x[s].x[0] = tc[s];
      x[s].x[1] = th[s];
    }
  }
  __device__ static void store_state(const KParams& p, long long i0, const Vec<2>* x) {
    float tc[S], th[S];
#pragma unroll
    for (int s = 0; s < S; ++s) {
      tc[s] = x[s].x[0];
      th[s] = x[s].x[1];
    }
    st_block<S>(p.out0 + i0, tc);
    st_block<S>(p.out1 + i0, th);
  }
};
template <typename PT, int S> struct Block1<kScanDiag, PT, S> {
  __device__ static void load_in(const KParams& p, long long b, long long t0, float (*vin)[2]) {
    float ta[S], tb[S];
    ld_block<float, S>(reinterpret_cast<const float*>(p.in0) + b * p.L + t0, ta);
    ld_block<float, S>(p.in1 + b * p.L + t0, tb);
#pragma unroll
    for (int s = 0; s < S; ++s) {
      vin[s][0] = ta[s];
      vin[s][1] = tb[s];
    }
  }
  __device__ static void load_state(const KParams& p, long long i0, Vec<1>* x) {
    float t[S];
    ld_block_cg<S>(p.out0 + i0, t);
#pragma unroll
    for (int s = 0; s < S; ++s) x[s].x[0] = t[s];
  }
  __device__ static void store_state(const KParams& p, long long i0, const Vec<1>* x) {
    float t[S];
#pragma unroll
    for (int s = 0; s < S; ++s) t[s] = x[s].x[0];
    st_block<S>(p.out0 + i0, t);
  }
};
template <typename PT, int S> struct Block1<kScanBlock2, PT, S> {
  __device__ static void load_in(const KParams& p, long long b, long long t0, float (*vin)[6]) {
    float ta[4 * S], tb[2 * S];
    ld_block<float, 4 * S>(reinterpret_cast<const float*>(p.in0) + (b * p.L + t0) * 4, ta);
    ld_block<float, 2 * S>(p.in1 + (b * p.L + t0) * 2, tb);
#pragma unroll
    for (int s = 0; s < S; ++s) {
#pragma unroll
      for (int i = 0; i < 4; ++i) vin[s][i] = ta[4 * s + i];
      vin[s][4] = tb[2 * s];
      vin[s][5] = tb[2 * s + 1];
    }
  }
  __device__ static void load_state(const KParams& p, long long i0, Vec<2>* x) {
    float t[2 * S];
    ld_block_cg<2 * S>(p.out0 + 2 * i0, t);
#pragma unroll
    for (int s = 0; s < S; ++s) {
      x[s].x[0] = t[2 * s];
      x[s].x[1] = t[2 * s + 1];
    }
  }
  __device__ static void store_state(const KParams& p, long long i0, const Vec<2>* x) {
    float t[2 * S];
#pragma unroll
    for (int s = 0; s < S; ++s) {
      t[2 * s] = x[s].x[0];
      t[2 * s + 1] = x[s].x[1];
    }
    st_block<2 * S>(p.out0 + 2 * i0, t);
  }
};

// Map of one step, from the inputs (scans) or from the cell at the iterate.
template <int OP> struct StepMap;
template <> struct StepMap<kScanDiag> {
  __device__ static Map<1> from_inputs(const float* v) {
    Map<1> m;
    m.m[0][0] = v[0];
    m.v[0] = v[1];
    return m;
  }
};
template <> struct StepMap<kScanBlock2> {
  __device__ static Map<2> from_inputs(const float* v) {
    Map<2> m;
    m.m[0][0] = v[0];
    m.m[0][1] = v[1];
    m.m[1][0] = v[2];
    m.m[1][1] = v[3];
    m.v[0] = v[4];
    m.v[1] = v[5];
    return m;
  }
};

// Newton linearisation of one step at the iterate:
//   map: x_t = J x_{t-1} + (f - J xprev),  rmax = max(rmax, |f - xcur|).
template <int OP>
__device__ __forceinline__ Map<OpT<OP>::NS> newton_step(const float* pin, const float* w,
                                                        const Vec<OpT<OP>::NS>& xprev,
                                                        const Vec<OpT<OP>::NS>& xcur,
                                                        float& rmax);
template <>
__device__ __forceinline__ Map<1> newton_step<kGru>(const float* pin, const float* w,
                                                    const Vec<1>& xprev, const Vec<1>& xcur,
                                                    float& rmax) {
  float f, J;
  gru_cell(pin, w, xprev.x[0], f, J);
  rmax = max_abs_nan(rmax, f - xcur.x[0]);
  Map<1> m;
  m.m[0][0] = J;
  m.v[0] = fmaf(-J, xprev.x[0], f);
  return m;
}
template <>
__device__ __forceinline__ Map<2> newton_step<kLstm>(const float* pin, const float* w,
                                                     const Vec<2>& xprev, const Vec<2>& xcur,
                                                     float& rmax) {
  float fc, fh, J[2][2];
  lstm_cell(pin, w, xprev.x[0], xprev.x[1], fc, fh, J);
  rmax = max_abs_nan(max_abs_nan(rmax, fc - xcur.x[0]), fh - xcur.x[1]);
  Map<2> m;
  m.m[0][0] = J[0][0];
  m.m[0][1] = J[0][1];
  m.m[1][0] = J[1][0];
  m.m[1][1] = J[1][1];
  m.v[0] = fc - fmaf(J[0][0], xprev.x[0], J[0][1] * xprev.x[1]);
  m.v[1] = fh - fmaf(J[1][0], xprev.x[0], J[1][1] * xprev.x[1]);
  return m;
}

// ---------------------------------------------------------------------------
// The kernel.
//
// Two ways to chain the time chunks of a tile (both exact, same arithmetic):
//  WALK = true   one CTA takes a whole tile and walks its chunks in time order;
//                the state entering chunk j at every iteration of the sweep is
//                the one chunk j-1 produced, kept in shared memory.  No traffic
//                between CTAs.  Used when there are enough tiles to fill the GPU.
//  WALK = false  a unit is one (tile, chunk); chunks of a tile run on different
//                CTAs at once and are chained by decoupled look-back through
//                global memory.  Used when the channels are few and the time
//                axis must provide the parallelism (e.g. one channel, 2^20 steps).
// ---------------------------------------------------------------------------
constexpr int kMaxWalkIters = 8;  // iterations per sweep kept in shared memory (WALK)

template <int OP, typename PT, int CW, int S, int MINB, bool WALK>
__global__ void __launch_bounds__(kThreads, MINB) pararnn_kernel(const KParams p) {
  using T_ = OpT<OP>;
  constexpr int NS = T_::NS;
  constexpr int NI = T_::NI;
  constexpr bool NEWTON = T_::newton;
  constexpr int NSEG = kThreads / CW;
  constexpr int TCH = NSEG * S;  // steps per chunk
  constexpr int WM = WALK ? kMaxWalkIters : 1;

  __shared__ Map<NS> s_wagg[kWarps][CW];
  __shared__ Vec<NS> s_carry[CW];
  __shared__ unsigned s_rmax[kWarps];
  __shared__ Vec<NS> s_inc[WALK ? 2 : 1][WM][CW];   // WALK: chunk-end state per iteration
  __shared__ Vec<NS> s_pend[WALK ? 2 : 1][CW];      // WALK: chunk-end state of the loaded iterate
  __shared__ unsigned s_racc[WM];                   // WALK: residual max per iteration
  __shared__ int s_unit;
  __shared__ int s_abort;
  __shared__ int s_done;

  const WaitCtx wctx{p.ctrl, p.status_dev, p.timeout_ns};
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int c = tid % CW;
  const int seg = tid / CW;
  const int nwork = WALK ? p.ntiles : p.nunits;

  int k0 = 0;
  int q = 0;
  if (tid == 0) {
    s_abort = 0;
  }
  __syncthreads();

  for (;; ++q) {
    const int m = NEWTON ? sweep_len(q, k0, p.m_first, p.m_next, p.max_iters) : 1;
    const unsigned epoch = (unsigned)(q + 1);

    for (;;) {  // work items of this sweep: tiles (WALK) or (tile, chunk) units
      if (tid == 0) {
        int u = (int)atomicAdd(&p.ticket[q], 1u);
        if (ld_volatile(&p.ctrl->abort) != 0u) u = nwork;
        s_unit = u;
      }
      if (WALK && tid < WM) s_racc[tid] = 0u;
      __syncthreads();
      const int item = s_unit;
      if (item >= nwork) break;

      const int jbeg = WALK ? 0 : item / p.ntiles;
      const int jend = WALK ? p.nchunks : jbeg + 1;
      const int tile = WALK ? item : item - jbeg * p.ntiles;
      const long long b = tile / p.ntd;
      const int td = tile - (int)b * p.ntd;
      const long long d = (long long)td * CW + c;
      const bool cvalid = d < p.D;
      const long long bd = b * p.D + d;

      float wv[NEWTON ? NI : 1];
      if constexpr (NEWTON) {
#pragma unroll
        for (int g = 0; g < NI; ++g) wv[g] = cvalid ? __ldg(p.w + (long long)g * p.D + d) : 0.0f;
      }

      for (int j = jbeg; j < jend; ++j) {
        const int u = j * p.ntiles + tile;  // unit index (look-back slots)
        const long long t0 = (long long)j * TCH + (long long)seg * S;
        const bool publish = (long long)u != p.stall_unit;

        // ---- stage this chunk's inputs in registers ------------------------
        // (D == 1 and aligned: the S steps are one contiguous block)
        bool blk = false;
        if constexpr (CW == 1) blk = p.vec1 && cvalid && t0 + S <= p.L;
        float vin[S][NI];
        if (blk) {
          if constexpr (CW == 1) Block1<OP, PT, S>::load_in(p, b, t0, vin);
        } else {
#pragma unroll
          for (int s = 0; s < S; ++s) {
            const long long t = t0 + s;
            if (cvalid && t < p.L) {
              IO<OP, PT>::load_in(p, (b * p.L + t) * p.D + d, b, t, d, vin[s]);
            } else {
#pragma unroll
              for (int i = 0; i < NI; ++i) vin[s][i] = 0.0f;
            }
          }
        }

        // ---- current iterate of the chunk and the state before each segment
        Vec<NS> x[S];
        Vec<NS> xb;  // state at t0 - 1 for the current iterate
#pragma unroll
        for (int i = 0; i < NS; ++i) xb.x[i] = 0.0f;
        if constexpr (NEWTON) {
          if (k0 == 0) {
#pragma unroll
            for (int s = 0; s < S; ++s)
#pragma unroll
              for (int i = 0; i < NS; ++i) x[s].x[i] = 0.0f;
            if (t0 == 0 && cvalid) IO<OP, PT>::init_state(p, bd, xb.x);
          } else {
            if (blk) {
              if constexpr (CW == 1) Block1<OP, PT, S>::load_state(p, b * p.L + t0, x);
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
            }
            if (cvalid) {
              if (t0 == 0) {
                IO<OP, PT>::init_state(p, bd, xb.x);
              } else if (seg == 0) {
                if constexpr (WALK) {
                  xb = s_pend[(j - 1) & 1][c];
                } else {
                  const float* src = p.bnd + ((size_t)((q - 1) & 1) * p.nunits + (u - p.ntiles)) *
                                                 (size_t)CW * NS + (size_t)c * NS;
#pragma unroll
                  for (int i = 0; i < NS; ++i) xb.x[i] = ldcg(src + i);
                }
              } else if (t0 - 1 < p.L) {
                IO<OP, PT>::load_state(p, (b * p.L + t0 - 1) * p.D + d, xb.x);
              }
            }
          }
          if constexpr (WALK) {
            // the loaded iterate's chunk end, for the next chunk's first segment
            if (seg == NSEG - 1) s_pend[j & 1][c] = x[S - 1];
          }
        }

        bool any_update = false;
        for (int kk = 0; kk < m; ++kk) {
          const int k = k0 + kk;
          const bool upd = !NEWTON || k < p.max_iters;

          // ---- step maps, residual, thread aggregate -----------------------
          Map<NS> mp[S];
          Map<NS> agg = map_identity<NS>();
          float rmax = 0.0f;
          Vec<NS> xp = xb;
#pragma unroll
          for (int s = 0; s < S; ++s) {
            const bool v = cvalid && (t0 + s) < p.L;
            if (v) {
              if constexpr (NEWTON) {
                mp[s] = newton_step<OP>(vin[s], wv, xp, x[s], rmax);
                xp = x[s];
              } else {
                mp[s] = StepMap<OP>::from_inputs(vin[s]);
              }
            } else {
              mp[s] = map_identity<NS>();
            }
            agg = compose(mp[s], agg);
          }
          unsigned rbits = 0u;
          if constexpr (NEWTON) rbits = __reduce_max_sync(0xffffffffu, __float_as_uint(rmax));

          if (!upd) {
            // residual-only iteration (k == max_iters): no solve, no update
            if constexpr (NEWTON) {
              if (lane == 0) s_rmax[warp] = rbits;
              __syncthreads();
              if (tid == 0) {
                unsigned r = s_rmax[0];
#pragma unroll
                for (int w2 = 1; w2 < kWarps; ++w2) r = max(r, s_rmax[w2]);
                if constexpr (WALK) {
                  s_racc[kk] = max(s_racc[kk], r);
                } else {
                  atomicMax(&p.rho_bits[k], r);
                }
              }
              __syncthreads();
            }
            continue;
          }
          any_update = true;

          // ---- segmented scan inside the warp (segments stride CW) ---------
          Map<NS> incl = agg;
          Map<NS> wexcl = map_identity<NS>();
          if constexpr (CW < 32) {
#pragma unroll
            for (int off = CW; off < 32; off <<= 1) {
              Map<NS> o = shfl_up_map(incl, off);
              if (lane >= off) incl = compose(incl, o);
            }
            Map<NS> e = shfl_up_map(incl, CW);
            if (lane >= CW) wexcl = e;
          }
          if (lane >= 32 - CW) s_wagg[warp][c] = incl;
          if constexpr (NEWTON) {
            if (lane == 0) s_rmax[warp] = rbits;
          }
          __syncthreads();

          // ---- chunk aggregate and the state carried into the chunk --------
          if (warp == 0) {
            Map<NS> cta = map_identity<NS>();
            if (lane < CW) {
#pragma unroll
              for (int w2 = 0; w2 < kWarps; ++w2) cta = compose(s_wagg[w2][c], cta);
            }
            if constexpr (NEWTON) {
              if (lane == 0) {
                unsigned r = s_rmax[0];
#pragma unroll
                for (int w2 = 1; w2 < kWarps; ++w2) r = max(r, s_rmax[w2]);
                if constexpr (WALK) {
                  s_racc[kk] = max(s_racc[kk], r);
                } else {
                  atomicMax(&p.rho_bits[k], r);
                }
              }
            }
            Vec<NS> carry;
            bool failed = false;
            if (j == 0) {
              if (lane < CW && cvalid) {
                IO<OP, PT>::init_state(p, bd, carry.x);
              } else {
#pragma unroll
                for (int i = 0; i < NS; ++i) carry.x[i] = 0.0f;
              }
            } else if constexpr (WALK) {
              carry = s_inc[(j - 1) & 1][kk][c];
            } else {
              constexpr int RW = Rec<NS>::kWords;
              unsigned long long* my_rec =
                  p.rec + (((size_t)kk * p.nunits + u) * CW + c) * RW;
              if (publish && lane < CW) publish_agg<NS>(my_rec, epoch, cta);
#pragma unroll
              for (int i = 0; i < NS; ++i) carry.x[i] = 0.0f;
              failed = !window_lookback<NS, CW>(p.rec + (size_t)kk * p.nunits * CW * RW,
                                                (size_t)CW * RW, u - p.ntiles, p.ntiles, epoch,
                                                carry, wctx);
            }
            const Vec<NS> xe = apply(cta, carry);
            if constexpr (WALK) {
              if (lane < CW) s_inc[j & 1][kk][c] = xe;
            } else {
              if (publish && !failed && lane < CW) {
                constexpr int RW = Rec<NS>::kWords;
                publish_inc<NS>(p.rec + (((size_t)kk * p.nunits + u) * CW + c) * RW, epoch, xe);
              }
            }
            if (lane < CW) s_carry[c] = carry;
            if (lane == 0 && failed) s_abort = 1;
          }
          // prefix of the earlier warps of this chunk, for this thread's channel
          Map<NS> wpre = map_identity<NS>();
          for (int w2 = 0; w2 < warp; ++w2) wpre = compose(s_wagg[w2][c], wpre);
          __syncthreads();

          // ---- carry in, apply the maps ------------------------------------
          const Vec<NS> xin = apply(wexcl, apply(wpre, s_carry[c]));
          Vec<NS> xr = xin;
#pragma unroll
          for (int s = 0; s < S; ++s) {
            xr = apply(mp[s], xr);
            x[s] = xr;
          }
          xb = xin;
          if (s_abort) break;
        }

        // ---- write the trajectory and the sweep boundary --------------------
        if (any_update || k0 == 0 || !NEWTON) {
          if (blk) {
            if constexpr (CW == 1) Block1<OP, PT, S>::store_state(p, b * p.L + t0, x);
          } else {
#pragma unroll
            for (int s = 0; s < S; ++s) {
              const long long t = t0 + s;
              if (cvalid && t < p.L) IO<OP, PT>::store_state(p, (b * p.L + t) * p.D + d, x[s].x);
            }
          }
        }
        if constexpr (NEWTON && !WALK) {
          if (seg == NSEG - 1) {
            float* dst =
                p.bnd + ((size_t)(q & 1) * p.nunits + u) * (size_t)CW * NS + (size_t)c * NS;
#pragma unroll
            for (int i = 0; i < NS; ++i) __stcg(dst + i, x[S - 1].x[i]);
          }
        }
        if (s_abort) break;
      }
      if constexpr (NEWTON && WALK) {
        __syncthreads();
        if (tid < m) atomicMax(&p.rho_bits[k0 + tid], s_racc[tid]);
      }
      if (s_abort) break;
      __syncthreads();  // s_unit and s_racc are rewritten for the next item
    }
    if (s_abort) break;

    if constexpr (!NEWTON) {
      break;
    } else {
      // every CTA takes the same decision from the same global residuals
      if (!grid_barrier(wctx)) {
        if (tid == 0) s_abort = 1;
        __syncthreads();
        break;
      }
      if (tid == 0) s_done = sweep_stops(p.rho_bits, k0, m, p.max_iters, p.tol);
      __syncthreads();
      if (s_done) break;
      k0 += m;
    }
  }

  // ---- report ---------------------------------------------------------------
  if constexpr (NEWTON) {
    if (blockIdx.x == 0 && tid == 0)
      write_solve_info(p.info, p.ctrl, p.rho_bits,
                       k0 + sweep_len(q, k0, p.m_first, p.m_next, p.max_iters) - 1, q + 1,
                       p.max_iters, p.tol, 0u);
  }
  // scans: a device-side error was written to status_dev by raise_error()
}

}  // namespace pararnn
