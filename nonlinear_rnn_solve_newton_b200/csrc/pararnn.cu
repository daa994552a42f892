// pararnn.cu -- C ABI of libpararnn.so (declared in include/pararnn.h).
//
// Host side: argument validation, the work decomposition (tile width along D,
// steps per thread, chunks), the workspace layout, and the launches of the
// kernel in pararnn_kernel.cuh.  Nothing here allocates, frees or synchronises:
// the caller owns every buffer and the stream.
#include <cuda_runtime.h>

#include <climits>
#include <cmath>
#include <cstdint>
#include <mutex>

#include <cudaTypedefs.h>

#include "pararnn.h"
#include "pararnn_bwd.cuh"
#include "pararnn_bwd_walk.cuh"
#include "pararnn_kernel.cuh"
#include "pararnn_mhgru.cuh"
#include "pararnn_mhgru2.cuh"
#include "pararnn_probe.cuh"
#include "pararnn_proj.cuh"
#include "pararnn_projsolve.cuh"
#include "pararnn_seq.cuh"
#include "pararnn_walk.cuh"

namespace pararnn {
namespace {

// Steps per thread for each operation (registers per thread grow with S and
// with the number of inputs per step).
// (Overridable at build time for tuning sweeps.)
#ifndef PARARNN_STEPS_SCAN_DIAG
#define PARARNN_STEPS_SCAN_DIAG 16
#endif
#ifndef PARARNN_STEPS_SCAN_BLOCK2
#define PARARNN_STEPS_SCAN_BLOCK2 8
#endif
#ifndef PARARNN_STEPS_GRU
#define PARARNN_STEPS_GRU 8
#endif
#ifndef PARARNN_STEPS_LSTM
#define PARARNN_STEPS_LSTM 4
#endif
// Steps per thread of the GRU look-back kernel on one-channel tiles (D = 1: long
// single-channel sequences, the DEER shape).  There a Newton iteration is bound
// by the look-back chain across the chunks in flight, so longer chunks (fewer of
// them) pay.  Measured on B200, B=16, L=2^20, D=1: 8 steps 0.336 ms, 16 steps
// 0.267 ms (123 registers, no spills).
#ifndef PARARNN_STEPS_GRU_NARROW
#define PARARNN_STEPS_GRU_NARROW 16
#endif
#ifndef PARARNN_MINB_SCAN
#define PARARNN_MINB_SCAN 2
#endif
#ifndef PARARNN_MINB_SOLVE
#define PARARNN_MINB_SOLVE 2
#endif
#ifndef PARARNN_WALK_STEPS_GRU
#define PARARNN_WALK_STEPS_GRU 16
#endif
#ifndef PARARNN_WALK_STEPS_LSTM
#define PARARNN_WALK_STEPS_LSTM 8
#endif
#ifndef PARARNN_WALK_STEPS_SCAN_DIAG
#define PARARNN_WALK_STEPS_SCAN_DIAG 16
#endif
#ifndef PARARNN_WALK_STEPS_SCAN_BLOCK2
#define PARARNN_WALK_STEPS_SCAN_BLOCK2 4
#endif
// Resident 8-warp CTAs per SM the walker's registers are held to: 3 where the
// staged chunk is small (scans, bf16 GRU), 2 for fp32 GRU and LSTM, whose
// larger per-thread state would otherwise spill (chosen by measurement).
#ifndef PARARNN_WALK_MINB
#define PARARNN_WALK_MINB 3
#endif
#ifndef PARARNN_WALK_MINB_WIDE
#define PARARNN_WALK_MINB_WIDE 2
#endif
// the same for the GRU solve's 32-channel walker, fp32 and bf16 gates
#ifndef PARARNN_WALK_MINB_GRU_F32
#define PARARNN_WALK_MINB_GRU_F32 PARARNN_WALK_MINB_WIDE
#endif
#ifndef PARARNN_WALK_MINB_GRU_BF16
#define PARARNN_WALK_MINB_GRU_BF16 PARARNN_WALK_MINB
#endif
constexpr int kWalkStepsGru = PARARNN_WALK_STEPS_GRU;
constexpr int kWalkStepsLstm = PARARNN_WALK_STEPS_LSTM;
constexpr int kWalkStepsScanDiag = PARARNN_WALK_STEPS_SCAN_DIAG;
constexpr int kWalkStepsScanBlock2 = PARARNN_WALK_STEPS_SCAN_BLOCK2;
constexpr int kWalkMinBlocks = PARARNN_WALK_MINB;
constexpr int kWalkMinBlocksWide = PARARNN_WALK_MINB_WIDE;
constexpr int kStepsScanDiag = PARARNN_STEPS_SCAN_DIAG;
constexpr int kStepsScanBlock2 = PARARNN_STEPS_SCAN_BLOCK2;
constexpr int kStepsGru = PARARNN_STEPS_GRU;
constexpr int kStepsLstm = PARARNN_STEPS_LSTM;
constexpr int kStepsGruNarrow = PARARNN_STEPS_GRU_NARROW;
// Resident CTAs per SM the register allocation is held to (launch bounds).
constexpr int kMinBlocksScan = PARARNN_MINB_SCAN;
constexpr int kMinBlocksSolve = PARARNN_MINB_SOLVE;
// Tiles from which one CTA per tile walking its chunks fills the GPU.
constexpr int kWalkMinTiles = 200;
// Below this many tiles the walker uses 16-warp CTAs.
constexpr int kWalkWideTiles = 512;
// Below this many 32-channel tiles (4 per SM on B200) the solves' walker uses
// 8-channel tiles, provided each tile is long enough for the better balance to
// outweigh the fixed cost of four times as many tiles (pipeline fill, the first
// stage's copy latency).  Measured on B200, GRU B=8 D=1024 with CUDA-graph
// replay, 8- vs 32-channel tiles: L=64 37 vs 21 us, 512 65 vs 51 us, 1024 99 vs
// 92 us, 1536 132 vs 128 us, 2048 164 vs 165 us, 3072 222 vs 238 us, 4096 289
// vs 311 us; the LSTM crosses over at the same length (1536: 289 vs 288 us,
// 2048: 358 vs 378 us).
constexpr int kWalkNarrowTiles = 4 * 148;
#ifndef PARARNN_NARROW_MIN_LEN
#define PARARNN_NARROW_MIN_LEN 2048
#endif
constexpr long long kWalkNarrowMinLen = PARARNN_NARROW_MIN_LEN;
// The solves' walker on 8-channel tiles.  A warp holds 8 channels x 4
// segments; with S steps per segment, segment k of a warp starts 24 S k words
// (GRU, fp32 rows of 3 gates) or 8 S k words (LSTM gate planes) into the stage,
// so an odd S puts the four segments on different shared-memory banks (S a
// multiple of 4 would make every read a 4-way conflict), and NW x 4 x S must
// stay within TMA's 256 rows per box.
// Measured on B200 (GRU, B=8, L=4096, D=1024): 4 warps x 13 steps 0.289 ms,
// 4 x 15 0.293 ms, 8 x 7 0.312 ms, 8 x 5 0.342 ms; 32-channel tiles 0.311 ms.
#ifndef PARARNN_NARROW_STEPS
#define PARARNN_NARROW_STEPS 13
#endif
#ifndef PARARNN_NARROW_WARPS
#define PARARNN_NARROW_WARPS 4
#endif
constexpr int kNarrowSteps = PARARNN_NARROW_STEPS;
// Resident-CTA targets (launch bounds) of the 8-channel walker.  Measured on
// B200 (B=8, L=4096, D=1024): the fp32 GRU walker at a target of 2 takes 108
// registers (4 CTAs per SM) and 288 us, at 4 it takes 96 (5 CTAs, the shared-
// memory limit) and 263 us, at 5 it takes 80 (still 5 CTAs) and 277 us; the
// LSTM walker at 2 takes 166 registers (3 CTAs) and 658 us, at 3 156 (3 CTAs)
// and 695 us, at 4 128 with spills (4 CTAs) and 690 us.
#ifndef PARARNN_NARROW_MINB_GRU
#define PARARNN_NARROW_MINB_GRU 4
#endif
#ifndef PARARNN_NARROW_MINB_GRU_BF16
#define PARARNN_NARROW_MINB_GRU_BF16 3
#endif
#ifndef PARARNN_NARROW_MINB_LSTM
#define PARARNN_NARROW_MINB_LSTM 2
#endif
constexpr int kNarrowMinBlocksGru = PARARNN_NARROW_MINB_GRU;
constexpr int kNarrowMinBlocksGruBf16 = PARARNN_NARROW_MINB_GRU_BF16;
constexpr int kNarrowMinBlocksLstm = PARARNN_NARROW_MINB_LSTM;
constexpr int kNarrowWarps = PARARNN_NARROW_WARPS;
static_assert(kNarrowWarps * 4 * kNarrowSteps <= 256, "TMA box rows");


constexpr int kStepsGruBwd = 8;
constexpr int kStepsLstmBwd = 4;
// Backward TMA walker, per cell: warps per CTA, steps per warp (a chunk is
// their product) and CTAs per SM for the register budget.  Measured on B200 at
// B=8, L=4096, D=1024: the GRU pass runs best with 32-step chunks (4 or 8
// warps alike), the LSTM pass (1.5x the bytes per step) with 72-step chunks of
// 12 warps and the full register file.
#ifndef PARARNN_BWD_WALK_WARPS_GRU
#define PARARNN_BWD_WALK_WARPS_GRU 8
#endif
#ifndef PARARNN_BWD_WALK_STEPS_GRU
#define PARARNN_BWD_WALK_STEPS_GRU 4
#endif
#ifndef PARARNN_BWD_WALK_MINB_GRU
#define PARARNN_BWD_WALK_MINB_GRU 2
#endif
#ifndef PARARNN_BWD_WALK_WARPS_LSTM
#define PARARNN_BWD_WALK_WARPS_LSTM 12
#endif
#ifndef PARARNN_BWD_WALK_STEPS_LSTM
#define PARARNN_BWD_WALK_STEPS_LSTM 6
#endif
#ifndef PARARNN_BWD_WALK_MINB_LSTM
#define PARARNN_BWD_WALK_MINB_LSTM 1
#endif

int steps_for(int op) {
  switch (op) {
    case kScanDiag: return kStepsScanDiag;
    case kScanBlock2: return kStepsScanBlock2;
    case kGru: return kStepsGru;
    case kGruBwd: return kStepsGruBwd;
    case kLstmBwd: return kStepsLstmBwd;
    default: return kStepsLstm;
  }
}
int walk_steps_for(int op) {
  switch (op) {
    case kScanDiag: return kWalkStepsScanDiag;
    case kScanBlock2: return kWalkStepsScanBlock2;
    case kGru: return kWalkStepsGru;
    default: return kWalkStepsLstm;
  }
}
int ns_for(int op) { return (op == kScanBlock2 || op == kLstm || op == kLstmBwd) ? 2 : 1; }
bool is_backward(int op) { return op == kGruBwd || op == kLstmBwd; }
// 64-bit words of one look-back record (aggregate, then chunk-end state).
int rec_words_for(int op) { return ns_for(op) == 2 ? Rec<2>::kWords : Rec<1>::kWords; }
bool is_newton(int op) { return op == kGru || op == kLstm; }

// Channels per tile: 32 (one warp row of 128 B for fp32) once D allows,
// otherwise the largest power of two not above D.
int tile_width(long long D) {
  int cw = 1;
  while (cw < 32 && (long long)cw * 2 <= D) cw *= 2;
  return cw;
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct Plan {
  bool walk = false;
  int S_walk = 0;   // steps per thread of the TMA walk kernel
  int NW_walk = 8;  // warps per CTA of the TMA walk kernel
  int CW_walk = 32; // channels per tile of the TMA walk kernel
  int op = 0, CW = 1, S = 1, T = 1, ntd = 0, ntiles = 0, nchunks = 0, nunits = 0;
  int m_first = 1, m_next = 1, mmax = 1, npasses = 1, max_iters = 0;
  size_t off_rho = 0, off_ticket = 0, off_rec = 0, zero_bytes = 0;
  size_t off_bnd = 0, total = 0;
  bool ok = false;
};

int count_sweeps(int m_first, int m_next, int max_iters) {
  int q = 0, k0 = 0;
  for (;;) {
    int m = sweep_len(q, k0, m_first, m_next, max_iters);
    ++q;
    if (k0 + m > max_iters) break;
    k0 += m;
  }
  return q;
}

Plan make_plan(int op, long long B, long long L, long long D, int max_iters,
               const pararnn_options_t* opts) {
  Plan pl;
  pl.op = op;
  if (B <= 0 || L <= 0 || D <= 0) return pl;
  if (is_newton(op) && (max_iters < 0 || max_iters > PARARNN_MAX_ITERS)) return pl;
  pl.CW = tile_width(D);
  pl.S = (op == kGru && pl.CW == 1) ? kStepsGruNarrow : steps_for(op);
  pl.T = (kThreads / pl.CW) * pl.S;
  long long ntd = (D + pl.CW - 1) / pl.CW;
  long long ntiles = B * ntd;
  long long nchunks = (L + pl.T - 1) / pl.T;
  if (ntiles > INT_MAX / 2 || nchunks > INT_MAX / 2 || ntiles * nchunks > INT_MAX / 2) return pl;
  pl.ntd = (int)ntd;
  pl.ntiles = (int)ntiles;
  pl.nchunks = (int)nchunks;
  pl.nunits = (int)(ntiles * nchunks);
  // Chain the chunks of a tile inside one CTA when the tiles alone fill the GPU
  // (about one tile per resident CTA or more); otherwise spread the chunks over
  // CTAs and chain them by look-back.
  const int regime = opts ? opts->regime : 0;
  if (regime == 1) {
    pl.walk = false;
  } else if (regime == 2) {
    pl.walk = true;
  } else {
    pl.walk = pl.nchunks > 1 && ntiles >= kWalkMinTiles;
    if (pl.nchunks == 1) pl.walk = true;
  }
  if (pl.walk && pl.CW == 32 && !is_backward(op)) {
    // the TMA walker cuts time into chunks of its own length
    pl.S_walk = walk_steps_for(op);
    const int want = opts ? opts->walk_warps : 0;
    // 16-warp CTAs only help the diagonal scan when tiles are few (measured on
    // B200); the solves and the 2x2 scan keep 8 warps.
    const bool wide = op == kScanDiag && ntiles < kWalkWideTiles;
    pl.NW_walk = (want == 4 || want == 8 || want == 16) ? want : (wide ? 16 : 8);
    // Tile width: 32-channel tiles leave the SMs unevenly loaded when there are
    // few of them per SM (256 tiles on 148 SMs: 108 SMs hold two, 40 hold one);
    // 8-channel tiles (a warp = 8 channels x 4 segments) cut the tail to < 2%.
    const int ww = opts ? opts->walk_width : 0;
    if (is_newton(op))
      pl.CW_walk = (ww == 8 || ww == 32) ? ww
                   : (ntiles < kWalkNarrowTiles && L >= kWalkNarrowMinLen ? 8 : 32);
    if (pl.CW_walk == 8) {
      pl.S_walk = kNarrowSteps;
      pl.NW_walk = kNarrowWarps;
    }
    const long long ntd_w = (D + pl.CW_walk - 1) / pl.CW_walk;
    if (B * ntd_w > INT_MAX / 2) return pl;
    long long tw = (long long)pl.NW_walk * (32 / pl.CW_walk) * pl.S_walk;
    long long nchunks_w = (L + tw - 1) / tw;
    if (nchunks_w > INT_MAX / 2) return pl;
  }
  if (is_newton(op)) {
    pl.max_iters = max_iters;
    // Iterations in the first sweep: Newton on these cells needs rho_0..rho_3
    // (GRU) or rho_0..rho_4 (LSTM, whose 2x2 coupling converges a step later)
    // for tol = 1e-4 at every workload measured, so one sweep usually suffices.
    int mf = (opts && opts->iters_first > 0) ? opts->iters_first : (op == kLstm ? 5 : 4);
    int mn = (opts && opts->iters_next > 0) ? opts->iters_next : 2;
    const int mcap = pl.walk ? kMaxWalkIters : PARARNN_MAX_ITERS + 1;
    if (mf > mcap) mf = mcap;
    if (mn > mcap) mn = mcap;
    pl.m_first = mf;
    pl.m_next = mn;
    pl.mmax = mf > mn ? mf : mn;
    if (pl.mmax > max_iters + 1) pl.mmax = max_iters + 1;
    pl.npasses = count_sweeps(mf, mn, max_iters);
  } else {
    pl.max_iters = 0;
    pl.m_first = pl.m_next = pl.mmax = 1;
    pl.npasses = 1;
  }
  const int NS = ns_for(op);
  size_t off = sizeof(Ctrl);
  pl.off_rho = off;
  off += sizeof(unsigned) * (size_t)(pl.max_iters + 1);
  pl.off_ticket = off;
  off += sizeof(unsigned) * (size_t)pl.npasses;
  off = align_up(off, 256);
  pl.off_rec = off;  // look-back records: zeroed with the control block
  if (!pl.walk) off += sizeof(unsigned long long) * (size_t)pl.mmax * pl.nunits * pl.CW *
                       (size_t)rec_words_for(op);
  off = align_up(off, 256);
  pl.zero_bytes = off;
  pl.off_bnd = off;
  if (!pl.walk && is_newton(op)) off += sizeof(float) * 2 * (size_t)pl.nunits * pl.CW * NS;
  pl.total = align_up(off, 256);
  pl.ok = true;
  return pl;
}

// ---------------------------------------------------------------------------
// Kernel selection by tile width.
// ---------------------------------------------------------------------------
template <int OP, typename PT, int S, int MINB, bool WALK>
const void* kernel_for_cw(int cw) {
  switch (cw) {
    case 1: return (const void*)pararnn_kernel<OP, PT, 1, S, MINB, WALK>;
    case 2: return (const void*)pararnn_kernel<OP, PT, 2, S, MINB, WALK>;
    case 4: return (const void*)pararnn_kernel<OP, PT, 4, S, MINB, WALK>;
    case 8: return (const void*)pararnn_kernel<OP, PT, 8, S, MINB, WALK>;
    case 16: return (const void*)pararnn_kernel<OP, PT, 16, S, MINB, WALK>;
    default: return (const void*)pararnn_kernel<OP, PT, 32, S, MINB, WALK>;
  }
}

template <int OP, typename PT, int S, int MINB>
const void* kernel_for(bool walk, int cw) {
  return walk ? kernel_for_cw<OP, PT, S, MINB, true>(cw) : kernel_for_cw<OP, PT, S, MINB, false>(cw);
}

const void* select_kernel(int op, bool bf16, bool walk, int cw) {
  switch (op) {
    case kScanDiag: return kernel_for<kScanDiag, float, kStepsScanDiag, kMinBlocksScan>(walk, cw);
    case kScanBlock2:
      return kernel_for<kScanBlock2, float, kStepsScanBlock2, kMinBlocksScan>(walk, cw);
    case kGru:
      if (cw == 1)
        return bf16 ? kernel_for<kGru, __nv_bfloat16, kStepsGruNarrow, kMinBlocksSolve>(walk, 1)
                    : kernel_for<kGru, float, kStepsGruNarrow, kMinBlocksSolve>(walk, 1);
      return bf16 ? kernel_for<kGru, __nv_bfloat16, kStepsGru, kMinBlocksSolve>(walk, cw)
                  : kernel_for<kGru, float, kStepsGru, kMinBlocksSolve>(walk, cw);
    default:
      return bf16 ? kernel_for<kLstm, __nv_bfloat16, kStepsLstm, kMinBlocksSolve>(walk, cw)
                  : kernel_for<kLstm, float, kStepsLstm, kMinBlocksSolve>(walk, cw);
  }
}

template <int OP, typename PT, int S, bool WALK>
const void* bwd_kernel_for_cw(int cw) {
  switch (cw) {
    case 1: return (const void*)pararnn_bwd_kernel<OP, PT, 1, S, 2, WALK>;
    case 2: return (const void*)pararnn_bwd_kernel<OP, PT, 2, S, 2, WALK>;
    case 4: return (const void*)pararnn_bwd_kernel<OP, PT, 4, S, 2, WALK>;
    case 8: return (const void*)pararnn_bwd_kernel<OP, PT, 8, S, 2, WALK>;
    case 16: return (const void*)pararnn_bwd_kernel<OP, PT, 16, S, 2, WALK>;
    default: return (const void*)pararnn_bwd_kernel<OP, PT, 32, S, 2, WALK>;
  }
}

template <int OP, int S>
const void* bwd_kernel_for(bool bf16, bool walk, int cw) {
  if (bf16)
    return walk ? bwd_kernel_for_cw<OP, __nv_bfloat16, S, true>(cw)
                : bwd_kernel_for_cw<OP, __nv_bfloat16, S, false>(cw);
  return walk ? bwd_kernel_for_cw<OP, float, S, true>(cw) : bwd_kernel_for_cw<OP, float, S, false>(cw);
}

// Backward TMA walker for an op and P dtype, with its dynamic shared memory,
// chunk length and threads per CTA.
template <int OP, typename PT, int S, int NW, int MINB>
const void* bwd_walk_kernel(size_t* smem, int* tch, int* threads) {
  *smem = 2 * (size_t)BwdStage<OP, PT, NW * S>::kPadded + 1024;  // + alignment slack
  *tch = NW * S;
  *threads = 32 * NW;
  return (const void*)pararnn_bwd_walk_kernel<OP, PT, S, NW, MINB>;
}

const void* select_bwd_walk_kernel(int op, bool bf16, size_t* smem, int* tch, int* threads) {
  constexpr int WG = PARARNN_BWD_WALK_WARPS_GRU, SG = PARARNN_BWD_WALK_STEPS_GRU,
                MG = PARARNN_BWD_WALK_MINB_GRU;
  constexpr int WL = PARARNN_BWD_WALK_WARPS_LSTM, SL = PARARNN_BWD_WALK_STEPS_LSTM,
                ML = PARARNN_BWD_WALK_MINB_LSTM;
  if (op == kGruBwd)
    return bf16 ? bwd_walk_kernel<kGruBwd, __nv_bfloat16, SG, WG, MG>(smem, tch, threads)
                : bwd_walk_kernel<kGruBwd, float, SG, WG, MG>(smem, tch, threads);
  return bf16 ? bwd_walk_kernel<kLstmBwd, __nv_bfloat16, SL, WL, ML>(smem, tch, threads)
              : bwd_walk_kernel<kLstmBwd, float, SL, WL, ML>(smem, tch, threads);
}

// Resident CTAs per SM for a kernel, cached per (device, kernel).
struct OccEntry {
  int dev;
  const void* fn;
  int per_sm;
  int nsm;
};
std::mutex g_occ_mu;
OccEntry g_occ[256];
int g_occ_n = 0;

cudaError_t resident_ctas(const void* fn, int threads, size_t dyn_smem, int* total) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  {
    std::lock_guard<std::mutex> lk(g_occ_mu);
    for (int i = 0; i < g_occ_n; ++i)
      if (g_occ[i].dev == dev && g_occ[i].fn == fn) {
        *total = g_occ[i].per_sm * g_occ[i].nsm;
        return cudaSuccess;
      }
  }
  int nsm = 0, per_sm = 0;
  e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, threads, dyn_smem);
  if (e != cudaSuccess) return e;
  {
    std::lock_guard<std::mutex> lk(g_occ_mu);
    if (g_occ_n < 256) g_occ[g_occ_n++] = OccEntry{dev, fn, per_sm, nsm};
  }
  *total = per_sm * nsm;
  return cudaSuccess;
}

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

// ---------------------------------------------------------------------------
// Tile-walking kernel with TMA staging (32-channel tiles).
// ---------------------------------------------------------------------------

template <int OP, typename PT, int S, int NW, int CW = 32>
size_t walk_smem_bytes() {
  constexpr unsigned b = Stage<OP, PT, NW * (32 / CW) * S, CW>::kBytes;
  return 2 * (size_t)((b + 1023u) / 1024u * 1024u) + 1024;  // + alignment slack
}

// Warps per CTA of the walker: 8, or 16 when the tiles are too few to fill the
// SMs with 8-warp CTAs (more warps per tile then hide more latency).
template <int OP, typename PT, int S, int MINB>
const void* walk_kernel_nw(int nw, size_t* smem) {
  if (nw == 16) {
    *smem = walk_smem_bytes<OP, PT, S, 16>();
    return (const void*)pararnn_walk_kernel<OP, PT, S, 16, (MINB + 1) / 2>;
  }
  if (nw == 4) {
    *smem = walk_smem_bytes<OP, PT, S, 4>();
    return (const void*)pararnn_walk_kernel<OP, PT, S, 4, 2 * MINB>;
  }
  *smem = walk_smem_bytes<OP, PT, S, 8>();
  return (const void*)pararnn_walk_kernel<OP, PT, S, 8, MINB>;
}

// The solves' walker on 8-channel tiles.
template <int OP, typename PT, int MINB>
const void* walk_kernel_narrow(size_t* smem) {
  *smem = walk_smem_bytes<OP, PT, kNarrowSteps, kNarrowWarps, 8>();
  return (const void*)pararnn_walk_kernel<OP, PT, kNarrowSteps, kNarrowWarps, MINB, 8>;
}

const void* select_walk_kernel(int op, bool bf16, int nw, int cw, size_t* smem) {
  if (cw == 8 && op == kGru)
    return bf16 ? walk_kernel_narrow<kGru, __nv_bfloat16, kNarrowMinBlocksGruBf16>(smem)
                : walk_kernel_narrow<kGru, float, kNarrowMinBlocksGru>(smem);
  if (cw == 8 && op == kLstm)
    return bf16 ? walk_kernel_narrow<kLstm, __nv_bfloat16, kNarrowMinBlocksLstm>(smem)
                : walk_kernel_narrow<kLstm, float, kNarrowMinBlocksLstm>(smem);
  switch (op) {
    case kScanDiag:
      return walk_kernel_nw<kScanDiag, float, kWalkStepsScanDiag, kWalkMinBlocks>(nw, smem);
    case kScanBlock2:
      return walk_kernel_nw<kScanBlock2, float, kWalkStepsScanBlock2, kWalkMinBlocks>(nw, smem);
    case kGru:
      return bf16 ? walk_kernel_nw<kGru, __nv_bfloat16, kWalkStepsGru, PARARNN_WALK_MINB_GRU_BF16>(
                        nw, smem)
                  : walk_kernel_nw<kGru, float, kWalkStepsGru, PARARNN_WALK_MINB_GRU_F32>(nw, smem);
    default:
      return bf16
                 ? walk_kernel_nw<kLstm, __nv_bfloat16, kWalkStepsLstm, kWalkMinBlocksWide>(nw, smem)
                 : walk_kernel_nw<kLstm, float, kWalkStepsLstm, kWalkMinBlocksWide>(nw, smem);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    else
      cudaGetLastError();
  });
  return g_encode;
}

// Row-major tensor [outer][mid][inner] (mid = 1 for 2-D), TMA box = inner x mid x rows.
// promo: the L2 promotion of the copies' DRAM reads.
bool encode_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, size_t esize,
                unsigned long long inner, unsigned long long mid, unsigned long long outer,
                unsigned box_inner, unsigned box_rows, unsigned box_mid = 0,
                CUtensorMapL2promotion promo = CU_TENSOR_MAP_L2_PROMOTION_L2_256B) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return false;
  CUresult r;
  const cuuint32_t estr[3] = {1, 1, 1};
  if (mid > 1) {
    const cuuint64_t dims[3] = {inner, mid, outer};
    const cuuint64_t strides[2] = {inner * esize, inner * mid * esize};
    const cuuint32_t box[3] = {box_inner, box_mid ? box_mid : (cuuint32_t)mid, box_rows};
    r = enc(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            promo, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  } else {
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {inner * esize};
    const cuuint32_t box[2] = {box_inner, box_rows};
    r = enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            promo, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  }
  return r == CUDA_SUCCESS;
}

// Tensor maps for the walk kernel, or false if the shapes or pointers do not
// meet TMA's rules (16-byte aligned base, row pitch a multiple of 16 bytes).
bool make_walk_maps(int op, bool bf16, const KParams& kp, int T, int CW, TmaMaps* tm) {
  const long long B = kp.B, L = kp.L, D = kp.D;
  if (D < CW || B * L >= (1LL << 31)) return false;
  const size_t es = bf16 ? 2 : 4;
  const CUtensorMapDataType dt =
      bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  const unsigned long long rows = (unsigned long long)(B * L);
  switch (op) {
    case kGru:
    case kLstm: {
      const int G = op == kGru ? 3 : 4;
      if (!aligned(kp.in0, 16) || (D * (long long)es) % 16 != 0) return false;
      // 8-channel LSTM tiles are staged one gate plane per copy
      const unsigned box_mid = (op == kLstm && CW == 8) ? 1u : 0u;
      // An 8-channel tile reads 32-byte row pieces.  With 256-byte promotion the
      // other seven tiles of each promoted block must use it before it leaves L2,
      // and at 5 CTAs per SM many do not: measured on B200 (GRU, B=8, L=4096,
      // D=1024, ncu) DRAM reads of 752 MB for 403 MB of gates, against 544 MB
      // with 64-byte promotion (663 MB at 128, 692 MB with none), all at the same
      // solve time; the LSTM 615 -> 573 MB for 537 MB of gates.
      const CUtensorMapL2promotion promo =
          CW == 8 ? CU_TENSOR_MAP_L2_PROMOTION_L2_64B : CU_TENSOR_MAP_L2_PROMOTION_L2_256B;
      return encode_map(&tm->in0, kp.in0, dt, es, D, G, rows, (unsigned)CW, T, box_mid, promo);
    }
    case kScanDiag:
      if (!aligned(kp.in0, 16) || !aligned(kp.in1, 16) || (D * 4) % 16 != 0) return false;
      return encode_map(&tm->in0, kp.in0, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, D, 1, rows, 32, T) &&
             encode_map(&tm->in1, kp.in1, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, D, 1, rows, 32, T);
    default:
      if (!aligned(kp.in0, 16) || !aligned(kp.in1, 16)) return false;
      return encode_map(&tm->in0, kp.in0, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, 4 * D, 1, rows,
                        128, T) &&
             encode_map(&tm->in1, kp.in1, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, 2 * D, 1, rows, 64,
                        T);
  }
}

// Tensor maps for the backward walker, or false if TMA's rules do not hold for
// every array it stages (16-byte aligned bases, row pitches a multiple of 16 B).
bool make_bwd_maps(int op, bool bf16, const BwdParams& bp, int T, BwdMaps* tm) {
  const long long B = bp.B, L = bp.L, D = bp.D;
  // (row coordinates and the per-chunk dP offsets are 32-bit in the kernel)
  if (D < 32 || D > (1LL << 24) || B * L >= (1LL << 31) || (D * 4) % 16 != 0) return false;
  const size_t es = bf16 ? 2 : 4;
  if ((D * (long long)es) % 16 != 0) return false;
  const int G = op == kGruBwd ? 3 : 4;
  const unsigned long long rows = (unsigned long long)(B * L);
  const CUtensorMapDataType f32 = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  const void* planes[4] = {bp.tr0, bp.tr1, bp.g0, bp.g1};
  CUtensorMap* maps[4] = {&tm->x0, &tm->x1, &tm->g0, &tm->g1};
  if (!aligned(bp.P, 16)) return false;
  if (!encode_map(&tm->P, bp.P, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : f32, es, D, G, rows,
                  32, T))
    return false;
  for (int i = 0; i < 4; ++i) {
    if (!planes[i]) continue;
    if (!aligned(planes[i], 16) || !encode_map(maps[i], planes[i], f32, 4, D, 1, rows, 32, T))
      return false;
  }
  return true;
}

// Empty problem: no equations, so the solve has converged at k = 0.
__global__ void empty_info_kernel(pararnn_solve_info_t* info) {
  info->iterations = 0;
  info->converged = 1;
  info->status = 0;
  info->updates = 0;
  info->passes = 0;
  info->reserved = 0;
  info->max_residual = 0.0f;
  for (int k = 0; k <= PARARNN_MAX_ITERS; ++k) info->rho[k] = 0.0f;
}

pararnn_status_t launch(const Plan& pl, KParams& kp, bool bf16, void* ws, size_t ws_bytes,
                        const pararnn_options_t* opts, cudaStream_t stream) {
  if (!ws || ws_bytes < pl.total || !aligned(ws, 256)) return PARARNN_ERR_WORKSPACE;
  char* base = static_cast<char*>(ws);
  kp.ctrl = reinterpret_cast<Ctrl*>(base);
  kp.rho_bits = reinterpret_cast<unsigned*>(base + pl.off_rho);
  kp.ticket = reinterpret_cast<unsigned*>(base + pl.off_ticket);
  kp.rec = reinterpret_cast<unsigned long long*>(base + pl.off_rec);
  // D == 1: a thread's S steps form one contiguous block; 16-byte vectors need
  // every array aligned and each block start on a 16-byte boundary (L % 8 == 0
  // covers the narrowest element, bf16 gate triples).
  kp.vec1 = kp.D == 1 && kp.L % 8 == 0 && aligned(kp.in0, 16) &&
            (!kp.in1 || aligned(kp.in1, 16)) && aligned(kp.out0, 16) &&
            (!kp.out1 || aligned(kp.out1, 16));
  kp.bnd = reinterpret_cast<float*>(base + pl.off_bnd);
  kp.ntd = pl.ntd;
  kp.ntiles = pl.ntiles;
  kp.nchunks = pl.nchunks;
  kp.nunits = pl.nunits;
  kp.max_iters = pl.max_iters;
  kp.m_first = pl.m_first;
  kp.m_next = pl.m_next;
  kp.mmax = pl.mmax;
  kp.timeout_ns = (opts && opts->wait_timeout_ns > 0) ? opts->wait_timeout_ns : 1000000000LL;
  kp.stall_unit = opts ? opts->debug_stall_unit : -1;

  // The TMA tile walker when the tiles are 32 wide and TMA's rules hold;
  // otherwise the general kernel (look-back or register-staged walk).
  TmaMaps tm;
  const int tch_w = pl.NW_walk * (32 / pl.CW_walk) * pl.S_walk;  // steps per walker chunk
  const bool tma_walk = pl.walk && pl.CW == 32 && pl.S_walk > 0 &&
                        make_walk_maps(pl.op, bf16, kp, tch_w, pl.CW_walk, &tm);
  const void* fn;
  size_t dyn_smem = 0;
  int threads = kThreads;
  if (tma_walk) {
    fn = select_walk_kernel(pl.op, bf16, pl.NW_walk, pl.CW_walk, &dyn_smem);
    kp.nchunks = (int)((kp.L + tch_w - 1) / tch_w);
    kp.ntd = (int)((kp.D + pl.CW_walk - 1) / pl.CW_walk);
    kp.ntiles = (int)(kp.B * kp.ntd);
    threads = 32 * pl.NW_walk;
  } else {
    fn = select_kernel(pl.op, bf16, pl.walk, pl.CW);
  }
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, fn) != cudaSuccess) {
    cudaGetLastError();
    return PARARNN_ERR_UNSUPPORTED;
  }
  if (dyn_smem > 0 &&
      cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn_smem) !=
          cudaSuccess) {
    cudaGetLastError();
    return PARARNN_ERR_CUDA;
  }
  int resident = 0;
  if (resident_ctas(fn, threads, dyn_smem, &resident) != cudaSuccess || resident <= 0) {
    cudaGetLastError();
    return PARARNN_ERR_CUDA;
  }
  const int nwork = pl.walk ? kp.ntiles : pl.nunits;
  int grid = nwork < resident ? nwork : resident;

  if (cudaMemsetAsync(ws, 0, pl.zero_bytes, stream) != cudaSuccess) return PARARNN_ERR_CUDA;
  if (kp.status_dev && cudaMemsetAsync(kp.status_dev, 0, sizeof(int32_t), stream) != cudaSuccess)
    return PARARNN_ERR_CUDA;

  void* args_plain[] = {&kp};
  void* args_tma[] = {&kp, &tm};
  void** args = tma_walk ? args_tma : args_plain;
  cudaError_t e;
  if (is_newton(pl.op)) {
    // The sweeps are separated by a grid barrier: all CTAs must be resident.
    e = cudaLaunchCooperativeKernel(fn, dim3(grid), dim3(threads), args, dyn_smem, stream);
  } else {
    // Scans wait only on smaller tickets, which are always held by running CTAs.
    e = cudaLaunchKernel(fn, dim3(grid), dim3(threads), args, dyn_smem, stream);
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    return PARARNN_ERR_CUDA;
  }
  return PARARNN_OK;
}

pararnn_status_t launch_bwd(const Plan& pl, BwdParams& bp, bool bf16, void* ws, size_t ws_bytes,
                            const pararnn_options_t* opts, cudaStream_t stream) {
  if (!ws || ws_bytes < pl.total || !aligned(ws, 256)) return PARARNN_ERR_WORKSPACE;
  char* base = static_cast<char*>(ws);
  bp.ctrl = reinterpret_cast<Ctrl*>(base);
  bp.ticket = reinterpret_cast<unsigned*>(base + pl.off_ticket);
  bp.rec = reinterpret_cast<unsigned long long*>(base + pl.off_rec);
  bp.ntd = pl.ntd;
  bp.ntiles = pl.ntiles;
  bp.nchunks = pl.nchunks;
  bp.nunits = pl.nunits;
  bp.timeout_ns = (opts && opts->wait_timeout_ns > 0) ? opts->wait_timeout_ns : 1000000000LL;
  bp.stall_unit = opts ? opts->debug_stall_unit : -1;
  // The TMA walker when the tiles are 32 wide and TMA's rules hold; otherwise
  // the general kernel (look-back or register-staged walk).
  BwdMaps tm;
  const void* fn = nullptr;
  size_t dyn_smem = 0;
  int tch = 0, walk_threads = 0;
  bool tma_walk = false;
  if (pl.walk && pl.CW == 32) {
    fn = select_bwd_walk_kernel(pl.op, bf16, &dyn_smem, &tch, &walk_threads);
    tma_walk = make_bwd_maps(pl.op, bf16, bp, tch, &tm);
  }
  if (tma_walk) {
    bp.nchunks = (int)((bp.L + tch - 1) / tch);
  } else {
    dyn_smem = 0;
    fn = pl.op == kGruBwd ? bwd_kernel_for<kGruBwd, kStepsGruBwd>(bf16, pl.walk, pl.CW)
                          : bwd_kernel_for<kLstmBwd, kStepsLstmBwd>(bf16, pl.walk, pl.CW);
  }
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, fn) != cudaSuccess) {
    cudaGetLastError();
    return PARARNN_ERR_UNSUPPORTED;
  }
  if (dyn_smem > 0 &&
      cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn_smem) !=
          cudaSuccess) {
    cudaGetLastError();
    return PARARNN_ERR_CUDA;
  }
  int resident = 0;
  const int threads = tma_walk ? walk_threads : kThreads;
  if (resident_ctas(fn, threads, dyn_smem, &resident) != cudaSuccess || resident <= 0) {
    cudaGetLastError();
    return PARARNN_ERR_CUDA;
  }
  const int nwork = pl.walk ? pl.ntiles : pl.nunits;
  const int grid = nwork < resident ? nwork : resident;
  const int G = pl.op == kGruBwd ? 3 : 4;
  if (cudaMemsetAsync(ws, 0, pl.zero_bytes, stream) != cudaSuccess ||
      cudaMemsetAsync(bp.da, 0, sizeof(float) * G * (size_t)bp.D, stream) != cudaSuccess)
    return PARARNN_ERR_CUDA;
  if (bp.status_dev && cudaMemsetAsync(bp.status_dev, 0, sizeof(int32_t), stream) != cudaSuccess)
    return PARARNN_ERR_CUDA;
  void* args_plain[] = {&bp};
  void* args_tma[] = {&bp, &tm};
  // Waits are only on smaller tickets, which running CTAs hold: no grid barrier.
  if (cudaLaunchKernel(fn, dim3(grid), dim3(threads), tma_walk ? args_tma : args_plain,
                       dyn_smem, stream) != cudaSuccess) {
    cudaGetLastError();
    return PARARNN_ERR_CUDA;
  }
  return PARARNN_OK;
}

}  // namespace
}  // namespace pararnn

using namespace pararnn;

extern "C" {

int32_t pararnn_version(void) { return PARARNN_VERSION; }

const char* pararnn_status_string(pararnn_status_t s) {
  switch (s) {
    case PARARNN_OK: return "ok";
    case PARARNN_ERR_INVALID_ARGUMENT: return "invalid argument";
    case PARARNN_ERR_UNSUPPORTED: return "unsupported device (libpararnn needs sm_100a)";
    case PARARNN_ERR_CUDA: return "CUDA runtime error";
    case PARARNN_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case PARARNN_ERR_NONFINITE: return "non-finite residual";
    case PARARNN_ERR_WORKSPACE: return "workspace missing, too small or misaligned";
  }
  return "unknown status";
}

size_t pararnn_workspace_size(pararnn_op_t op, int64_t B, int64_t L, int64_t D, int32_t max_iters,
                              const pararnn_options_t* opts) {
  if ((int)op == 6) {  // multi-head GRU: control block + one residual word per iteration
    if (max_iters < 0 || max_iters > PARARNN_MAX_ITERS) return 0;
    return (sizeof(Ctrl) + 4 * (size_t)(max_iters + 1) + 255) / 256 * 256;
  }
  if ((int)op == 8) {  // strided multi-head GRU: + the heads' stride offsets (H = D / 8)
    if (max_iters < 0 || max_iters > PARARNN_MAX_ITERS || D < 0 || D % 8 != 0) return 0;
    const size_t base = (sizeof(Ctrl) + 4 * (size_t)(max_iters + 1) + 255) / 256 * 256;
    return base + (4 * (size_t)(D / 8 + 2) + 255) / 256 * 256;
  }
  if ((int)op == 7) {  // projected GRU solve: control block, residuals, no look-back records
    if (max_iters < 0 || max_iters > PARARNN_MAX_ITERS) return 0;
    return (sizeof(Ctrl) + 4 * (size_t)(max_iters + 1) + 255) / 256 * 256;
  }
  if ((int)op < 0 || (int)op > 5) return 0;
  if (B == 0 || L == 0 || D == 0) return 256;
  Plan pl = make_plan((int)op, B, L, D, max_iters, opts);
  return pl.ok ? pl.total : 0;
}

static pararnn_status_t scan_common(int op, const float* A, const float* b, const float* x0,
                                    float* x, int64_t B, int64_t L, int64_t D, void* ws,
                                    size_t ws_bytes, int32_t* status_dev,
                                    const pararnn_options_t* opts, void* stream) {
  if (B < 0 || L < 0 || D < 0) return PARARNN_ERR_INVALID_ARGUMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (B == 0 || L == 0 || D == 0) {
    if (status_dev && cudaMemsetAsync(status_dev, 0, sizeof(int32_t), st) != cudaSuccess)
      return PARARNN_ERR_CUDA;
    return PARARNN_OK;
  }
  if (!A || !b || !x) return PARARNN_ERR_INVALID_ARGUMENT;
  if (op == kScanBlock2) {
    if (!aligned(A, 16) || !aligned(b, 8) || !aligned(x, 8) || (x0 && !aligned(x0, 8)))
      return PARARNN_ERR_INVALID_ARGUMENT;
  } else {
    if (!aligned(A, 4) || !aligned(b, 4) || !aligned(x, 4) || (x0 && !aligned(x0, 4)))
      return PARARNN_ERR_INVALID_ARGUMENT;
  }
  Plan pl = make_plan(op, B, L, D, 0, opts);
  if (!pl.ok) return PARARNN_ERR_INVALID_ARGUMENT;
  KParams kp = {};
  kp.in0 = A;
  kp.in1 = b;
  kp.x0a = x0;
  kp.out0 = x;
  kp.B = B;
  kp.L = L;
  kp.D = D;
  kp.status_dev = status_dev;
  return launch(pl, kp, false, ws, ws_bytes, opts, st);
}

pararnn_status_t pararnn_scan_diag(const float* A, const float* b, const float* h0, float* h,
                                   int64_t B, int64_t L, int64_t D, void* ws, size_t ws_bytes,
                                   int32_t* status_dev, const pararnn_options_t* opts,
                                   void* stream) {
  return scan_common(kScanDiag, A, b, h0, h, B, L, D, ws, ws_bytes, status_dev, opts, stream);
}

pararnn_status_t pararnn_scan_block2(const float* A, const float* b, const float* x0, float* x,
                                     int64_t B, int64_t L, int64_t D, void* ws, size_t ws_bytes,
                                     int32_t* status_dev, const pararnn_options_t* opts,
                                     void* stream) {
  return scan_common(kScanBlock2, A, b, x0, x, B, L, D, ws, ws_bytes, status_dev, opts, stream);
}

static pararnn_status_t solve_common(int op, const void* P, pararnn_dtype_t p_dtype,
                                     const float* a, const float* x0a, const float* x0b,
                                     float* out0, float* out1, int64_t B, int64_t L, int64_t D,
                                     float tol, int32_t max_iters, void* ws, size_t ws_bytes,
                                     pararnn_solve_info_t* info, const pararnn_options_t* opts,
                                     void* stream) {
  if (B < 0 || L < 0 || D < 0) return PARARNN_ERR_INVALID_ARGUMENT;
  if (!info || !aligned(info, 4)) return PARARNN_ERR_INVALID_ARGUMENT;
  if (max_iters < 0 || max_iters > PARARNN_MAX_ITERS) return PARARNN_ERR_INVALID_ARGUMENT;
  if (!(tol >= 0.0f)) return PARARNN_ERR_INVALID_ARGUMENT;  // rejects NaN too
  if (p_dtype != PARARNN_F32 && p_dtype != PARARNN_BF16) return PARARNN_ERR_INVALID_ARGUMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (B == 0 || L == 0 || D == 0) {
    empty_info_kernel<<<1, 1, 0, st>>>(info);
    return cudaGetLastError() == cudaSuccess ? PARARNN_OK : PARARNN_ERR_CUDA;
  }
  if (!P || !a || !out0 || (op == kLstm && !out1)) return PARARNN_ERR_INVALID_ARGUMENT;
  const size_t esz = p_dtype == PARARNN_BF16 ? 2 : 4;
  if (!aligned(P, esz) || !aligned(a, 4) || !aligned(out0, 4) || (out1 && !aligned(out1, 4)) ||
      (x0a && !aligned(x0a, 4)) || (x0b && !aligned(x0b, 4)))
    return PARARNN_ERR_INVALID_ARGUMENT;
  Plan pl = make_plan(op, B, L, D, max_iters, opts);
  if (!pl.ok) return PARARNN_ERR_INVALID_ARGUMENT;
  KParams kp = {};
  kp.in0 = P;
  kp.w = a;
  kp.x0a = x0a;
  kp.x0b = x0b;
  kp.out0 = out0;
  kp.out1 = out1;
  kp.B = B;
  kp.L = L;
  kp.D = D;
  kp.tol = tol;
  kp.info = info;
  return launch(pl, kp, p_dtype == PARARNN_BF16, ws, ws_bytes, opts, st);
}

pararnn_status_t pararnn_solve_gru(const void* P, pararnn_dtype_t p_dtype, const float* a,
                                   const float* h0, float* h, int64_t B, int64_t L, int64_t D,
                                   float tol, int32_t max_iters, void* ws, size_t ws_bytes,
                                   pararnn_solve_info_t* info, const pararnn_options_t* opts,
                                   void* stream) {
  return solve_common(kGru, P, p_dtype, a, h0, nullptr, h, nullptr, B, L, D, tol, max_iters, ws,
                      ws_bytes, info, opts, stream);
}

pararnn_status_t pararnn_solve_lstm(const void* P, pararnn_dtype_t p_dtype, const float* a,
                                    const float* c0, const float* h0, float* c, float* h,
                                    int64_t B, int64_t L, int64_t D, float tol, int32_t max_iters,
                                    void* ws, size_t ws_bytes, pararnn_solve_info_t* info,
                                    const pararnn_options_t* opts, void* stream) {
  return solve_common(kLstm, P, p_dtype, a, c0, h0, c, h, B, L, D, tol, max_iters, ws, ws_bytes,
                      info, opts, stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free ParaGRU solve.
//
// Some callers cannot allocate device memory at the point where they solve:
// code whose device memory is entirely reserved by another allocator, a
// framework plug-in interface that hands over inputs and outputs but no
// workspace, or a latency-critical loop where an allocation (which may
// synchronise the device) is not allowed.  For them the scratch the kernel
// needs lives in the library itself: one file-scope device array of
// PARARNN_NOALLOC_SCRATCH_BYTES, which every GPU that loads the library holds
// until the process exits.
// ---------------------------------------------------------------------------
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[PARARNN_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
struct NoallocSlot {
  void* ptr;                 // device address of the array in that context
  unsigned long long ctx_id; // the driver's unique id of the context it was resolved in
};
NoallocSlot g_noalloc[kMaxDevices] = {};

// The driver's id of the calling thread's current context (0 if there is none
// or the driver does not offer the query).  Ids are never reused, so a context
// created after cudaDeviceReset has a new one even if its handle repeats.
unsigned long long current_context_id() {
  static PFN_cuCtxGetCurrent_v4000 get_cur = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_cur = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f);
    f = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(f);
    cudaGetLastError();
  });
  if (!get_cur || !get_id) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_cur(&ctx) != CUDA_SUCCESS || !ctx) return 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of the scratch array on the current device.  The name of the
// array is only a host-side stand-in and must never be handed to a kernel: the
// address is looked up with the device current, on the first call on that
// device, and again whenever the device's context has changed since (a
// cudaDeviceReset ends the context the cached address belonged to).
pararnn_status_t noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return PARARNN_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  NoallocSlot& slot = g_noalloc[dev];
  const unsigned long long id = current_context_id();
  if (!slot.ptr || id == 0 || id != slot.ctx_id) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return PARARNN_ERR_CUDA;
    }
    slot.ptr = p;
    // the lookup made the device's primary context current if none was
    slot.ctx_id = id != 0 ? id : current_context_id();
  }
  *out = slot.ptr;
  return PARARNN_OK;
}

}  // namespace

extern "C" pararnn_status_t pararnn_solve_gru_noalloc(const void* P, pararnn_dtype_t p_dtype,
                                                      const float* a, const float* h0, float* h,
                                                      int64_t B, int64_t L, int64_t D, float tol,
                                                      int32_t max_iters,
                                                      pararnn_solve_info_t* info,
                                                      const pararnn_options_t* opts,
                                                      void* stream) {
  if (B < 0 || L < 0 || D < 0) return PARARNN_ERR_INVALID_ARGUMENT;
  const size_t need = pararnn_workspace_size(PARARNN_OP_GRU, B, L, D, max_iters, opts);
  if (need == 0) return PARARNN_ERR_INVALID_ARGUMENT;
  if (need > (size_t)PARARNN_NOALLOC_SCRATCH_BYTES) return PARARNN_ERR_WORKSPACE;
  void* scratch = nullptr;
  pararnn_status_t st = noalloc_scratch(&scratch);
  if (st != PARARNN_OK) return st;
  return pararnn_solve_gru(P, p_dtype, a, h0, h, B, L, D, tol, max_iters, scratch,
                           (size_t)PARARNN_NOALLOC_SCRATCH_BYTES, info, opts, stream);
}

// ---------------------------------------------------------------------------
// Backward pass.
// ---------------------------------------------------------------------------
static pararnn_status_t backward_common(int op, const void* P, pararnn_dtype_t p_dtype,
                                        const float* a, const float* x0a, const float* x0b,
                                        const float* tr0, const float* tr1, const float* g0,
                                        const float* g1, float* dP, float* da, float* d0a,
                                        float* d0b, int64_t B, int64_t L, int64_t D, void* ws,
                                        size_t ws_bytes, int32_t* status_dev,
                                        const pararnn_options_t* opts, void* stream) {
  if (B < 0 || L < 0 || D < 0) return PARARNN_ERR_INVALID_ARGUMENT;
  if (p_dtype != PARARNN_F32 && p_dtype != PARARNN_BF16) return PARARNN_ERR_INVALID_ARGUMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int G = op == kGruBwd ? 3 : 4;
  if (B == 0 || L == 0 || D == 0) {
    // no steps: every gradient is zero
    if (da && D > 0 && cudaMemsetAsync(da, 0, sizeof(float) * G * (size_t)D, st) != cudaSuccess)
      return PARARNN_ERR_CUDA;
    if (B > 0 && D > 0) {
      if (d0a && cudaMemsetAsync(d0a, 0, sizeof(float) * (size_t)(B * D), st) != cudaSuccess)
        return PARARNN_ERR_CUDA;
      if (d0b && cudaMemsetAsync(d0b, 0, sizeof(float) * (size_t)(B * D), st) != cudaSuccess)
        return PARARNN_ERR_CUDA;
    }
    if (status_dev && cudaMemsetAsync(status_dev, 0, sizeof(int32_t), st) != cudaSuccess)
      return PARARNN_ERR_CUDA;
    return PARARNN_OK;
  }
  if (!P || !a || !tr0 || !dP || !da) return PARARNN_ERR_INVALID_ARGUMENT;
  if (op == kGruBwd && !g0) return PARARNN_ERR_INVALID_ARGUMENT;
  if (op == kLstmBwd && (!tr1 || (!g0 && !g1))) return PARARNN_ERR_INVALID_ARGUMENT;
  const size_t esz = p_dtype == PARARNN_BF16 ? 2 : 4;
  const void* ptrs4[] = {a, x0a, x0b, tr0, tr1, g0, g1, dP, da, d0a, d0b};
  for (const void* q : ptrs4)
    if (q && !aligned(q, 4)) return PARARNN_ERR_INVALID_ARGUMENT;
  if (!aligned(P, esz)) return PARARNN_ERR_INVALID_ARGUMENT;
  Plan pl = make_plan(op, B, L, D, 0, opts);
  if (!pl.ok) return PARARNN_ERR_INVALID_ARGUMENT;
  BwdParams bp = {};
  bp.P = P;
  bp.w = a;
  bp.x0a = x0a;
  bp.x0b = x0b;
  bp.tr0 = tr0;
  bp.tr1 = tr1;
  bp.g0 = g0;
  bp.g1 = g1;
  bp.dP = dP;
  bp.da = da;
  bp.d0a = d0a;
  bp.d0b = d0b;
  bp.B = B;
  bp.L = L;
  bp.D = D;
  bp.status_dev = status_dev;
  return launch_bwd(pl, bp, p_dtype == PARARNN_BF16, ws, ws_bytes, opts, st);
}

extern "C" pararnn_status_t pararnn_solve_gru_backward(
    const void* P, pararnn_dtype_t p_dtype, const float* a, const float* h0, const float* h,
    const float* dh, float* dP, float* da, float* dh0, int64_t B, int64_t L, int64_t D, void* ws,
    size_t ws_bytes, int32_t* status_dev, const pararnn_options_t* opts, void* stream) {
  return backward_common(kGruBwd, P, p_dtype, a, h0, nullptr, h, nullptr, dh, nullptr, dP, da,
                         dh0, nullptr, B, L, D, ws, ws_bytes, status_dev, opts, stream);
}

extern "C" pararnn_status_t pararnn_solve_lstm_backward(
    const void* P, pararnn_dtype_t p_dtype, const float* a, const float* c0, const float* h0,
    const float* c, const float* h, const float* dc, const float* dh, float* dP, float* da,
    float* dc0, float* dh0, int64_t B, int64_t L, int64_t D, void* ws, size_t ws_bytes,
    int32_t* status_dev, const pararnn_options_t* opts, void* stream) {
  return backward_common(kLstmBwd, P, p_dtype, a, c0, h0, c, h, dc, dh, dP, da, dc0, dh0, B, L, D,
                         ws, ws_bytes, status_dev, opts, stream);
}

// ---------------------------------------------------------------------------
// Sequential application on the GPU: one step (decode) and the full rollout.
// ---------------------------------------------------------------------------
static pararnn_status_t seq_common(bool rollout, int op, const void* P, pararnn_dtype_t p_dtype,
                                   const float* a, const float* x0a, const float* x0b,
                                   float* out0, float* out1, int64_t B, int64_t L, int64_t D,
                                   void* stream) {
  if (B < 0 || L < 0 || D < 0) return PARARNN_ERR_INVALID_ARGUMENT;
  if (p_dtype != PARARNN_F32 && p_dtype != PARARNN_BF16) return PARARNN_ERR_INVALID_ARGUMENT;
  if (B == 0 || L == 0 || D == 0) return PARARNN_OK;
  if (!P || !a || !out0 || (op == kLstm && !out1)) return PARARNN_ERR_INVALID_ARGUMENT;
  const size_t esz = p_dtype == PARARNN_BF16 ? 2 : 4;
  const void* ptrs[] = {a, x0a, x0b, out0, out1};
  for (const void* q : ptrs)
    if (q && !aligned(q, 4)) return PARARNN_ERR_INVALID_ARGUMENT;
  if (!aligned(P, esz)) return PARARNN_ERR_INVALID_ARGUMENT;
  if (B * D > (1LL << 40)) return PARARNN_ERR_INVALID_ARGUMENT;
  SeqParams sp = {P, a, x0a, x0b, out0, out1, B, L, D};
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool bf16 = p_dtype == PARARNN_BF16;
  const long long n = B * D;
  if (rollout) {
    const int threads = 128;
    const unsigned blocks = (unsigned)((n + threads - 1) / threads);
    // one channel per batch row: each thread stages its own contiguous inputs
    const long long G = op == kGru ? 3 : 4;
    if (D == 1 && aligned(P, 16) && (L * G * (long long)esz) % 16 == 0) {
      const int t1 = 64;
      const unsigned b1 = (unsigned)((B + t1 - 1) / t1);
      if (op == kGru) {
        if (bf16)
          pararnn_rollout_seq1_kernel<kGru, __nv_bfloat16, 16><<<b1, t1, 0, st>>>(sp);
        else
          pararnn_rollout_seq1_kernel<kGru, float, 16><<<b1, t1, 0, st>>>(sp);
      } else {
        if (bf16)
          pararnn_rollout_seq1_kernel<kLstm, __nv_bfloat16, 8><<<b1, t1, 0, st>>>(sp);
        else
          pararnn_rollout_seq1_kernel<kLstm, float, 8><<<b1, t1, 0, st>>>(sp);
      }
      return cudaGetLastError() == cudaSuccess ? PARARNN_OK : PARARNN_ERR_CUDA;
    }
    // inputs staged through shared memory when each warp's channels are one
    // contiguous row segment (D % 32 == 0) and the rows are 16-byte aligned
    if (D % 32 == 0 && aligned(P, 16)) {
      if (op == kGru) {
        if (bf16)
          pararnn_rollout_staged_kernel<kGru, __nv_bfloat16, 16><<<blocks, threads, 0, st>>>(sp);
        else
          pararnn_rollout_staged_kernel<kGru, float, 16><<<blocks, threads, 0, st>>>(sp);
      } else {
        if (bf16)
          pararnn_rollout_staged_kernel<kLstm, __nv_bfloat16, 8><<<blocks, threads, 0, st>>>(sp);
        else
          pararnn_rollout_staged_kernel<kLstm, float, 8><<<blocks, threads, 0, st>>>(sp);
      }
      return cudaGetLastError() == cudaSuccess ? PARARNN_OK : PARARNN_ERR_CUDA;
    }
    if (op == kGru) {
      if (bf16)
        pararnn_rollout_kernel<kGru, __nv_bfloat16, 16><<<blocks, threads, 0, st>>>(sp);
      else
        pararnn_rollout_kernel<kGru, float, 16><<<blocks, threads, 0, st>>>(sp);
    } else {
      if (bf16)
        pararnn_rollout_kernel<kLstm, __nv_bfloat16, 8><<<blocks, threads, 0, st>>>(sp);
      else
        pararnn_rollout_kernel<kLstm, float, 8><<<blocks, threads, 0, st>>>(sp);
    }
  } else {
    const int threads = 256;
    long long blocks = (n + threads - 1) / threads;
    if (blocks > 148 * 16) blocks = 148 * 16;
    if (op == kGru) {
      if (bf16)
        pararnn_step_kernel<kGru, __nv_bfloat16><<<(unsigned)blocks, threads, 0, st>>>(sp);
      else
        pararnn_step_kernel<kGru, float><<<(unsigned)blocks, threads, 0, st>>>(sp);
    } else {
      if (bf16)
        pararnn_step_kernel<kLstm, __nv_bfloat16><<<(unsigned)blocks, threads, 0, st>>>(sp);
      else
        pararnn_step_kernel<kLstm, float><<<(unsigned)blocks, threads, 0, st>>>(sp);
    }
  }
  if (cudaGetLastError() != cudaSuccess) return PARARNN_ERR_CUDA;
  return PARARNN_OK;
}

extern "C" pararnn_status_t pararnn_step_gru(const void* P, pararnn_dtype_t p_dtype,
                                             const float* a, const float* h_prev, float* h_next,
                                             int64_t B, int64_t D, void* stream) {
  return seq_common(false, kGru, P, p_dtype, a, h_prev, nullptr, h_next, nullptr, B, 1, D,
                    stream);
}

extern "C" pararnn_status_t pararnn_step_lstm(const void* P, pararnn_dtype_t p_dtype,
                                              const float* a, const float* c_prev,
                                              const float* h_prev, float* c_next, float* h_next,
                                              int64_t B, int64_t D, void* stream) {
  return seq_common(false, kLstm, P, p_dtype, a, c_prev, h_prev, c_next, h_next, B, 1, D, stream);
}

extern "C" pararnn_status_t pararnn_rollout_gru(const void* P, pararnn_dtype_t p_dtype,
                                                const float* a, const float* h0, float* h,
                                                int64_t B, int64_t L, int64_t D, void* stream) {
  return seq_common(true, kGru, P, p_dtype, a, h0, nullptr, h, nullptr, B, L, D, stream);
}

extern "C" pararnn_status_t pararnn_rollout_lstm(const void* P, pararnn_dtype_t p_dtype,
                                                 const float* a, const float* c0, const float* h0,
                                                 float* c, float* h, int64_t B, int64_t L,
                                                 int64_t D, void* stream) {
  return seq_common(true, kLstm, P, p_dtype, a, c0, h0, c, h, B, L, D, stream);
}

extern "C" pararnn_status_t pararnn_rollout_mhgru(const void* P, pararnn_dtype_t p_dtype,
                                                  const float* U, const float* h0, float* h,
                                                  int64_t B, int64_t L, int64_t H, void* stream) {
  using namespace pararnn;
  if (B < 0 || L < 0 || H < 0) return PARARNN_ERR_INVALID_ARGUMENT;
  if (p_dtype != PARARNN_F32 && p_dtype != PARARNN_BF16) return PARARNN_ERR_INVALID_ARGUMENT;
  if (B == 0 || L == 0 || H == 0) return PARARNN_OK;
  if (!P || !U || !h) return PARARNN_ERR_INVALID_ARGUMENT;
  const size_t esz = p_dtype == PARARNN_BF16 ? 2 : 4;
  if (!aligned(P, esz) || !aligned(U, 4) || (h0 && !aligned(h0, 4)) || !aligned(h, 4))
    return PARARNN_ERR_INVALID_ARGUMENT;
  if (B * H > (1LL << 31) / 8 || H > (1LL << 27)) return PARARNN_ERR_INVALID_ARGUMENT;
  MhSeqParams sp = {P, U, h0, h, B, L, H};
  const int threads = 64;  // 8 sequences per CTA
  const unsigned blocks = (unsigned)((B * H * 8 + threads - 1) / threads);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // inputs staged through shared memory when a warp's 4 heads are 32 contiguous
  // channels of one batch row (H % 4 == 0) and the rows are 16-byte aligned
  const bool staged = H % 4 == 0 && aligned(P, 16);
  if (p_dtype == PARARNN_BF16) {
    if (staged)
      pararnn_rollout_mhgru_kernel<__nv_bfloat16, 16, true><<<blocks, threads, 0, st>>>(sp);
    else
      pararnn_rollout_mhgru_kernel<__nv_bfloat16, 8, false><<<blocks, threads, 0, st>>>(sp);
  } else {
    if (staged)
      pararnn_rollout_mhgru_kernel<float, 16, true><<<blocks, threads, 0, st>>>(sp);
    else
      pararnn_rollout_mhgru_kernel<float, 8, false><<<blocks, threads, 0, st>>>(sp);
  }
  return cudaGetLastError() == cudaSuccess ? PARARNN_OK : PARARNN_ERR_CUDA;
}

// One decode step of the multi-head GRU is its rollout over one time step.
extern "C" pararnn_status_t pararnn_step_mhgru(const void* P, pararnn_dtype_t p_dtype,
                                               const float* U, const float* h_prev,
                                               float* h_next, int64_t B, int64_t H,
                                               void* stream) {
  return pararnn_rollout_mhgru(P, p_dtype, U, h_prev, h_next, B, 1, H, stream);
}

// ---------------------------------------------------------------------------
// Input projection P = x W^T + bias (tcgen05 tensor cores).
// ---------------------------------------------------------------------------
namespace pararnn {
namespace {

#ifndef PARARNN_PROJ_STAGES
#define PARARNN_PROJ_STAGES 4
#endif
constexpr int kProjStages = PARARNN_PROJ_STAGES;
#ifndef PARARNN_PROJ_PAIRS
#define PARARNN_PROJ_PAIRS 1
#endif
#ifndef PARARNN_PROJ2_STAGES
#define PARARNN_PROJ2_STAGES 6
#endif
constexpr bool kProjPairs = PARARNN_PROJ_PAIRS != 0;
constexpr int kProj2Stages = PARARNN_PROJ2_STAGES;

// K = 0: P is the bias broadcast over rows (or zero).
__global__ void proj_fill_kernel(const float* bias, void* out, long long M, long long N,
                                 int out_bf16) {
  const long long n = M * N;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const float v = bias ? bias[i % N] : 0.0f;
    if (out_bf16)
      static_cast<__nv_bfloat16*>(out)[i] = __float2bfloat16_rn(v);
    else
      static_cast<float*>(out)[i] = v;
  }
}

// bf16 row-major [outer][inner] operand, box = 64 (one 128-byte swizzle row) x rows.
bool encode_map_sw128(CUtensorMap* m, const void* base, unsigned long long inner,
                      unsigned long long outer, unsigned box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {inner * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// P [M, N] (fp32 or bf16) for the epilogue's tensor stores: box = 128 bytes of
// columns x 32 rows, 128-byte swizzle.
bool encode_map_out(CUtensorMap* m, void* base, unsigned long long N, unsigned long long M,
                    bool bf16) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return false;
  const size_t es = bf16 ? 2 : 4;
  const cuuint64_t dims[2] = {N, M};
  const cuuint64_t strides[1] = {N * es};
  const cuuint32_t box[2] = {(cuuint32_t)(128 / es), 32};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2,
             base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace
}  // namespace pararnn

extern "C" pararnn_status_t pararnn_input_projection(const void* x, const void* W,
                                                     const float* bias, void* P,
                                                     pararnn_dtype_t p_dtype, int64_t M,
                                                     int64_t N, int64_t K, int32_t* status_dev,
                                                     void* stream) {
  if (M < 0 || N < 0 || K < 0) return PARARNN_ERR_INVALID_ARGUMENT;
  if (p_dtype != PARARNN_F32 && p_dtype != PARARNN_BF16) return PARARNN_ERR_INVALID_ARGUMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (status_dev && cudaMemsetAsync(status_dev, 0, sizeof(int32_t), st) != cudaSuccess)
    return PARARNN_ERR_CUDA;
  if (M == 0 || N == 0) return PARARNN_OK;
  if (!P || N % 8 != 0 || K % 8 != 0 || M >= (1LL << 31) || N >= (1LL << 31) ||
      K >= (1LL << 31))
    return PARARNN_ERR_INVALID_ARGUMENT;
  if (!aligned(P, 16) || (bias && !aligned(bias, 16))) return PARARNN_ERR_INVALID_ARGUMENT;
  const int out_bf16 = p_dtype == PARARNN_BF16 ? 1 : 0;
  if (K == 0) {
    long long blocks = (M * N + 255) / 256;
    if (blocks > 148 * 16) blocks = 148 * 16;
    proj_fill_kernel<<<(unsigned)blocks, 256, 0, st>>>(bias, P, M, N, out_bf16);
    return cudaGetLastError() == cudaSuccess ? PARARNN_OK : PARARNN_ERR_CUDA;
  }
  if (!x || !W || !aligned(x, 16) || !aligned(W, 16)) return PARARNN_ERR_INVALID_ARGUMENT;
  const long long ntm = (M + kProjBM - 1) / kProjBM, ntn = (N + kProjBN - 1) / kProjBN;
  if (ntm * ntn >= (1LL << 31)) return PARARNN_ERR_INVALID_ARGUMENT;

  ProjMaps tm;
  if (!encode_map_sw128(&tm.x, x, (unsigned long long)K, (unsigned long long)M, kProjBM) ||
      !encode_map_out(&tm.p, P, (unsigned long long)N, (unsigned long long)M, out_bf16 != 0))
    return PARARNN_ERR_INVALID_ARGUMENT;
  ProjParams pp;
  pp.bias = bias;
  pp.out = P;
  pp.M = (int)M;
  pp.N = (int)N;
  pp.K = (int)K;
  pp.ntn = (int)ntn;
  pp.out_bf16 = out_bf16;
  pp.status_dev = status_dev;
  pp.timeout_ns = 1000000000LL;
  void* args[] = {&pp, &tm};

  // CTA pairs (tcgen05 cta_group::2, 256 x 256 tiles) up to K = 2048, one CTA
  // per 128 x 256 tile above.  Measured on B200, same box, alternating: K = 1024
  // pairs 0.177 ms vs 0.193 ms; K = 4096 (power-capped) pairs 4-10% slower.
  if (kProjPairs && K <= 2048) {
    const void* fn2 = out_bf16 ? (const void*)pararnn_proj2_kernel<kProj2Stages, true>
                               : (const void*)pararnn_proj2_kernel<kProj2Stages, false>;
    const size_t smem2 = proj2_smem_bytes<kProj2Stages>();
    cudaFuncAttributes fa2;
    int nclusters = 0;
    if (cudaFuncGetAttributes(&fa2, fn2) == cudaSuccess &&
        cudaFuncSetAttribute(fn2, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem2) ==
            cudaSuccess &&
        encode_map_sw128(&tm.w, W, (unsigned long long)K, (unsigned long long)N, kProjBN / 2)) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(2 * 74);
      cfg.blockDim = dim3(kProjThreads);
      cfg.dynamicSmemBytes = smem2;
      cfg.stream = st;
      if (cudaOccupancyMaxActiveClusters(&nclusters, fn2, &cfg) != cudaSuccess) nclusters = 0;
    }
    cudaGetLastError();
    if (nclusters > 0) {
      const long long ntiles2 = ((M + 2 * kProjBM - 1) / (2 * kProjBM)) * ntn;
      const unsigned pairs = (unsigned)(ntiles2 < nclusters ? ntiles2 : nclusters);
      if (cudaLaunchKernel(fn2, dim3(2 * pairs), dim3(kProjThreads), args, smem2, st) ==
          cudaSuccess)
        return PARARNN_OK;
      cudaGetLastError();
    }
  }

  const void* fn = out_bf16 ? (const void*)pararnn_proj_kernel<kProjStages, true>
                            : (const void*)pararnn_proj_kernel<kProjStages, false>;
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, fn) != cudaSuccess) {
    cudaGetLastError();
    return PARARNN_ERR_UNSUPPORTED;
  }
  const size_t smem = proj_smem_bytes<kProjStages>();
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess) {
    cudaGetLastError();
    return PARARNN_ERR_CUDA;
  }
  if (!encode_map_sw128(&tm.w, W, (unsigned long long)K, (unsigned long long)N, kProjBN))
    return PARARNN_ERR_INVALID_ARGUMENT;
  // persistent: one CTA per SM (the ring and both accumulators fill an SM)
  int resident = 0;
  if (resident_ctas(fn, kProjThreads, smem, &resident) != cudaSuccess || resident <= 0) {
    cudaGetLastError();
    return PARARNN_ERR_CUDA;
  }
  const long long ntiles = ntm * ntn;
  const unsigned grid = (unsigned)(ntiles < resident ? ntiles : resident);
  if (cudaLaunchKernel(fn, dim3(grid), dim3(kProjThreads), args, smem, st) != cudaSuccess) {
    cudaGetLastError();
    return PARARNN_ERR_CUDA;
  }
  return PARARNN_OK;
}

// ---------------------------------------------------------------------------
// Multi-head GRU (dense 8x8 blocks).
// ---------------------------------------------------------------------------
namespace pararnn {
namespace {

// Prefix offsets of the heads' strides (each capped at L: a stride of L or more
// makes every step depend on h0 alone) for the multi-head kernel's work units:
// offs[g] = sum of the capped strides before head g, offs[H] = their total,
// offs[H + 1] = 1 if some stride is below 1.  One warp.
__global__ void mh_stride_offsets_kernel(const int32_t* strides, int* offs, long long H,
                                         long long L) {
  const int lane = threadIdx.x;
  const long long per = (H + 31) / 32;
  const long long g0 = lane * per;
  const long long g1 = g0 + per < H ? g0 + per : H;
  long long sum = 0;
  int bad = 0;
  for (long long g = g0; g < g1; ++g) {
    const long long sg = strides[g];
    if (sg < 1) bad = 1;
    sum += sg < 1 ? 1 : (sg < L ? sg : L);
  }
  long long incl = sum;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const long long v = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += v;
  }
  long long acc = incl - sum;
  for (long long g = g0; g < g1; ++g) {
    offs[g] = (int)acc;
    const long long sg = strides[g];
    acc += sg < 1 ? 1 : (sg < L ? sg : L);
  }
  if (lane == 31) offs[H] = (int)incl;
  bad = __any_sync(0xffffffffu, bad);
  if (lane == 0) offs[H + 1] = bad;
}

size_t mh_offsets_at(int32_t max_iters) {
  return (sizeof(Ctrl) + 4 * (size_t)(max_iters + 1) + 255) / 256 * 256;
}

pararnn_status_t mhgru_common(const void* P, pararnn_dtype_t p_dtype, const float* U,
                              const int32_t* strides, const float* h0, float* h, int64_t B,
                              int64_t L, int64_t H, float tol, int32_t max_iters, void* ws,
                              size_t ws_bytes, pararnn_solve_info_t* info,
                              const pararnn_options_t* opts, void* stream) {
  if (B < 0 || L < 0 || H < 0) return PARARNN_ERR_INVALID_ARGUMENT;
  if (!info || !aligned(info, 4)) return PARARNN_ERR_INVALID_ARGUMENT;
  if (max_iters < 0 || max_iters > PARARNN_MAX_ITERS) return PARARNN_ERR_INVALID_ARGUMENT;
  if (!(tol >= 0.0f)) return PARARNN_ERR_INVALID_ARGUMENT;
  if (p_dtype != PARARNN_F32 && p_dtype != PARARNN_BF16) return PARARNN_ERR_INVALID_ARGUMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (B == 0 || L == 0 || H == 0) {
    empty_info_kernel<<<1, 1, 0, st>>>(info);
    return cudaGetLastError() == cudaSuccess ? PARARNN_OK : PARARNN_ERR_CUDA;
  }
  if (!P || !U || !h) return PARARNN_ERR_INVALID_ARGUMENT;
  if (!aligned(P, 16) || !aligned(U, 4) || !aligned(h, 16) || (h0 && !aligned(h0, 4)))
    return PARARNN_ERR_INVALID_ARGUMENT;
  if (B * H > (1LL << 40) || L > (1LL << 40)) return PARARNN_ERR_INVALID_ARGUMENT;
  // with strides, the work units of a batch row (sum of the capped strides) stay below 2^31
  if (strides && (!aligned(strides, 4) || H * L >= (1LL << 31))) return PARARNN_ERR_INVALID_ARGUMENT;
  const size_t need = pararnn_workspace_size(
      strides ? PARARNN_OP_MHGRU_STRIDED : PARARNN_OP_MHGRU, B, L, 8 * H, max_iters, opts);
  if (!ws || ws_bytes < need || !aligned(ws, 256)) return PARARNN_ERR_WORKSPACE;

  // Layout: one lane per time segment holding whole 8x8 maps, a warp per
  // sequence (regime 1), or 8 lanes per head and segment, a CTA per sequence
  // (regime 2).  Automatic: the first without strides, the second with them.
  // Measured on B200 (B=8, L=4096, 128 heads, fp32): unstrided 2.63 vs 3.17 ms;
  // strides 2^(g mod 8) 6.53 vs 5.42 ms.
  const int layout = opts ? opts->regime : 0;
  const bool lane_maps = layout == 1 || (layout != 2 && !strides);
  const bool bf = p_dtype == PARARNN_BF16;
  const void* fn =
      lane_maps ? (bf ? (const void*)pararnn_mhgru_kernel<__nv_bfloat16>
                      : (const void*)pararnn_mhgru_kernel<float>)
                : (bf ? (const void*)pararnn_mhgru2_kernel<__nv_bfloat16>
                      : (const void*)pararnn_mhgru2_kernel<float>);
  const size_t kMhSmem =
      lane_maps ? (bf ? mh_smem_bytes<__nv_bfloat16>() : mh_smem_bytes<float>())
                : (bf ? sizeof(Mh2Smem<__nv_bfloat16>) : sizeof(Mh2Smem<float>));
  const int mh_threads = lane_maps ? 32 * kMhWarps : kMh2Threads;
  const int units_per_cta = lane_maps ? kMhWarps : 1;
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, fn) != cudaSuccess) {
    cudaGetLastError();
    return PARARNN_ERR_UNSUPPORTED;
  }
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kMhSmem) !=
      cudaSuccess) {
    cudaGetLastError();
    return PARARNN_ERR_CUDA;
  }
  int resident = 0;
  if (resident_ctas(fn, mh_threads, kMhSmem, &resident) != cudaSuccess || resident <= 0) {
    cudaGetLastError();
    return PARARNN_ERR_CUDA;
  }
  // with strides the unit count is known on the device only: every resident CTA runs
  const long long units = B * H;
  const long long want = (units + units_per_cta - 1) / units_per_cta;
  const int grid = strides ? resident : (int)(want < resident ? want : resident);

  MhParams mp;
  mp.P = P;
  mp.U = U;
  mp.h0 = h0;
  mp.h = h;
  mp.B = B;
  mp.L = L;
  mp.H = H;
  mp.tol = tol;
  mp.max_iters = max_iters;
  mp.ctrl = static_cast<Ctrl*>(ws);
  mp.rho_bits = reinterpret_cast<unsigned*>(static_cast<char*>(ws) + sizeof(Ctrl));
  int* offs = strides ? reinterpret_cast<int*>(static_cast<char*>(ws) + mh_offsets_at(max_iters))
                      : nullptr;
  mp.offs = offs;
  mp.info = info;
  mp.status_dev = nullptr;
  mp.timeout_ns = (opts && opts->wait_timeout_ns > 0) ? opts->wait_timeout_ns : 1000000000LL;
  if (cudaMemsetAsync(ws, 0, need, st) != cudaSuccess) return PARARNN_ERR_CUDA;
  if (strides) {
    mh_stride_offsets_kernel<<<1, 32, 0, st>>>(strides, offs, H, L);
    if (cudaGetLastError() != cudaSuccess) return PARARNN_ERR_CUDA;
  }
  // no update at all: the result is the initial iterate h^0 = 0
  if (max_iters == 0 &&
      cudaMemsetAsync(h, 0, sizeof(float) * (size_t)(B * L * 8 * H), st) != cudaSuccess)
    return PARARNN_ERR_CUDA;
  void* args[] = {&mp};
  if (cudaLaunchCooperativeKernel(fn, dim3(grid), dim3(mh_threads), args, kMhSmem, st) !=
      cudaSuccess) {
    cudaGetLastError();
    return PARARNN_ERR_CUDA;
  }
  return PARARNN_OK;
}

}  // namespace
}  // namespace pararnn

extern "C" pararnn_status_t pararnn_solve_mhgru(const void* P, pararnn_dtype_t p_dtype,
                                                const float* U, const float* h0, float* h,
                                                int64_t B, int64_t L, int64_t H, float tol,
                                                int32_t max_iters, void* ws, size_t ws_bytes,
                                                pararnn_solve_info_t* info,
                                                const pararnn_options_t* opts, void* stream) {
  return pararnn::mhgru_common(P, p_dtype, U, nullptr, h0, h, B, L, H, tol, max_iters, ws,
                               ws_bytes, info, opts, stream);
}

extern "C" pararnn_status_t pararnn_solve_mhgru_strided(
    const void* P, pararnn_dtype_t p_dtype, const float* U, const int32_t* strides,
    const float* h0, float* h, int64_t B, int64_t L, int64_t H, float tol, int32_t max_iters,
    void* ws, size_t ws_bytes, pararnn_solve_info_t* info, const pararnn_options_t* opts,
    void* stream) {
  if (!strides && B > 0 && L > 0 && H > 0) return PARARNN_ERR_INVALID_ARGUMENT;
  return pararnn::mhgru_common(P, p_dtype, U, strides, h0, h, B, L, H, tol, max_iters, ws,
                               ws_bytes, info, opts, stream);
}

// ---------------------------------------------------------------------------
// Throughput probes (measured peaks for the rooflines).
// ---------------------------------------------------------------------------
extern "C" pararnn_status_t pararnn_probe_rate(int32_t pipe, int32_t iters, float* sink,
                                               int64_t* ops, void* stream) {
  using namespace pararnn;
  if ((pipe != 0 && pipe != 1) || iters <= 0 || !sink || !ops)
    return PARARNN_ERR_INVALID_ARGUMENT;
  const void* fn = pipe == 0 ? (const void*)pararnn_probe_kernel<0>
                             : (const void*)pararnn_probe_kernel<1>;
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, fn) != cudaSuccess) {
    cudaGetLastError();
    return PARARNN_ERR_UNSUPPORTED;
  }
  int total = 0;
  if (resident_ctas(fn, kProbeThreads, 0, &total) != cudaSuccess || total <= 0) {
    cudaGetLastError();
    return PARARNN_ERR_CUDA;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (pipe == 0)
    pararnn_probe_kernel<0><<<total, kProbeThreads, 0, st>>>(iters, sink);
  else
    pararnn_probe_kernel<1><<<total, kProbeThreads, 0, st>>>(iters, sink);
  if (cudaGetLastError() != cudaSuccess) return PARARNN_ERR_CUDA;
  const int64_t per_step = pipe == 0 ? 2 : 1;
  *ops = (int64_t)total * kProbeThreads * (int64_t)iters * kProbeUnroll * kProbeChains * per_step;
  return PARARNN_OK;
}

// ---------------------------------------------------------------------------
// Projected ParaGRU solve: input projection on the tensor cores fused with the
// Newton walk (P never reaches HBM).
// ---------------------------------------------------------------------------
namespace pararnn {
namespace {

#ifndef PARARNN_PS_STAGES
#define PARARNN_PS_STAGES 5
#endif
#ifndef PARARNN_PS_STAGES2
#define PARARNN_PS_STAGES2 4
#endif
constexpr int kPsStages = PARARNN_PS_STAGES;    // one walker group
constexpr int kPsStages2 = PARARNN_PS_STAGES2;  // two walker groups (two staged chunks)

// W [3 D, K] bf16 viewed as 3 gate blocks of D rows: {K, D, 3}, box {64, 32, 3},
// 128-byte swizzle (the box lands as 96 consecutive swizzled 128-byte rows).
bool encode_map_w3(CUtensorMap* m, const void* W, unsigned long long K, unsigned long long D) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[3] = {K, D, 3};
  const cuuint64_t strides[2] = {K * 2, D * K * 2};
  const cuuint32_t box[3] = {64, (cuuint32_t)kPsCW, 3};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(W), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace
}  // namespace pararnn

extern "C" pararnn_status_t pararnn_solve_gru_projected(
    const void* x, const void* W, const float* bias, const float* a, const float* h0, float* h,
    int64_t B, int64_t L, int64_t D, int64_t K, float tol, int32_t max_iters, void* ws,
    size_t ws_bytes, pararnn_solve_info_t* info, const pararnn_options_t* opts, void* stream) {
  using namespace pararnn;
  if (B < 0 || L < 0 || D < 0 || K < 0) return PARARNN_ERR_INVALID_ARGUMENT;
  if (!info || !aligned(info, 4)) return PARARNN_ERR_INVALID_ARGUMENT;
  if (max_iters < 0 || max_iters > PARARNN_MAX_ITERS) return PARARNN_ERR_INVALID_ARGUMENT;
  if (!(tol >= 0.0f)) return PARARNN_ERR_INVALID_ARGUMENT;  // rejects NaN too
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (B == 0 || L == 0 || D == 0) {
    empty_info_kernel<<<1, 1, 0, st>>>(info);
    return cudaGetLastError() == cudaSuccess ? PARARNN_OK : PARARNN_ERR_CUDA;
  }
  if (!x || !W || !a || !h) return PARARNN_ERR_INVALID_ARGUMENT;
  if (K == 0 || K % 8 != 0 || K >= (1LL << 31) || B * L >= (1LL << 31) || D >= (1LL << 30))
    return PARARNN_ERR_INVALID_ARGUMENT;
  if (!aligned(x, 16) || !aligned(W, 16) || (bias && !aligned(bias, 4)) || !aligned(a, 4) ||
      (h0 && !aligned(h0, 4)) || !aligned(h, 4))
    return PARARNN_ERR_INVALID_ARGUMENT;
  const size_t need = pararnn_workspace_size((pararnn_op_t)7, B, L, D, max_iters, opts);
  if (!ws || ws_bytes < need || !aligned(ws, 256)) return PARARNN_ERR_WORKSPACE;

  PsMaps tm;
  if (!encode_map_sw128(&tm.x, x, (unsigned long long)K, (unsigned long long)(B * L), kPsBM) ||
      !encode_map_w3(&tm.w, W, (unsigned long long)K, (unsigned long long)D))
    return PARARNN_ERR_INVALID_ARGUMENT;

  PsParams pp;
  pp.bias = bias;
  pp.w = a;
  pp.h0 = h0;
  pp.h = h;
  pp.B = B;
  pp.L = L;
  pp.D = D;
  pp.K = (int)K;
  pp.ntd = (int)((D + kPsCW - 1) / kPsCW);
  pp.nitems = (int)(B * pp.ntd);
  pp.nchunks = (int)((L + kPsBM - 1) / kPsBM);
  pp.tol = tol;
  pp.max_iters = max_iters;
  int mf = (opts && opts->iters_first > 0) ? opts->iters_first : 4;
  int mn = (opts && opts->iters_next > 0) ? opts->iters_next : 2;
  if (mf > kMaxWalkIters) mf = kMaxWalkIters;
  if (mn > kMaxWalkIters) mn = kMaxWalkIters;
  pp.m_first = mf;
  pp.m_next = mn;
  pp.ctrl = static_cast<Ctrl*>(ws);
  pp.rho_bits = reinterpret_cast<unsigned*>(static_cast<char*>(ws) + sizeof(Ctrl));
  pp.info = info;
  pp.timeout_ns = (opts && opts->wait_timeout_ns > 0) ? opts->wait_timeout_ns : 1000000000LL;
  if (B * (long long)pp.ntd >= (1LL << 31) || L / kPsBM >= (1LL << 30))
    return PARARNN_ERR_INVALID_ARGUMENT;

  // walker groups: two (two items per CTA at once) unless opts->regime = 1;
  // measured on B200 two were faster at every K from 256 to 4096
  const bool two = !(opts && opts->regime == 1);
  const void* fn = two ? (const void*)pararnn_projsolve_kernel<kPsStages2, 2>
                       : (const void*)pararnn_projsolve_kernel<kPsStages, 1>;
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, fn) != cudaSuccess) {
    cudaGetLastError();
    return PARARNN_ERR_UNSUPPORTED;
  }
  const size_t smem = two ? ps_smem_bytes<kPsStages2, 2>() : ps_smem_bytes<kPsStages, 1>();
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess) {
    cudaGetLastError();
    return PARARNN_ERR_CUDA;
  }
  int resident = 0;
  if (resident_ctas(fn, kPsThreads, smem, &resident) != cudaSuccess || resident <= 0) {
    cudaGetLastError();
    return PARARNN_ERR_CUDA;
  }
  const int grid = pp.nitems < resident ? pp.nitems : resident;
  if (cudaMemsetAsync(ws, 0, need, st) != cudaSuccess) return PARARNN_ERR_CUDA;
  void* args[] = {&pp, &tm};
  // sweeps are separated by a grid barrier: every CTA must be resident
  if (cudaLaunchCooperativeKernel(fn, dim3(grid), dim3(kPsThreads), args, smem, st) !=
      cudaSuccess) {
    cudaGetLastError();
    return PARARNN_ERR_CUDA;
  }
  return PARARNN_OK;
}
