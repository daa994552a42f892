#!/usr/bin/env python
"""Benchmark of the ParaGRU Newton solve (and the diagonal affine scan) on B200.

One step = one complete Newton solve, all iterations, of the LM-width ParaGRU
layer: B=8, L=8192, D=4096, bf16 projected gate inputs P ~ N(0,1), fp32 state,
Jacobians and scan, a ~ U(-0.5,0.5), h0 = 0, tol 1e-4, max 32 iterations.  The
same run times the diagonal affine scan at that width (B=8, L=8192, D=4096,
fp32: the scan HBM GB/s half of the metric) and, as extra keys, the fp32 solve
and scan at B=8, L=4096, D=1024.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload lm|gru_l|deer|gru_s|lstm|...]

Under torchrun (N > 1) every rank solves its own independent batch (weak
scaling, no data-path collective); the time is the max over ranks.  Rank 0
prints one JSON line.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from tests import inputs  # noqa: E402  (seeded synthetic inputs only)

METRIC = "Newton-solve channel-steps/sec (B*L*D) and scan HBM GB/s, % of B200 HBM peak"
UNIT = "channel-steps/s"
SMS = 148
MUFU_PER_STEP = {"gru": 6, "lstm": 10}   # (ex2 + rcp) per sigmoid/tanh, per channel-step
# multi-head GRU, per channel-step and Newton evaluation: gate matvecs 24 +
# Jacobian 24 + b_t 8 + map composition (8x8 product + matvec) 72 = 128 FMA
MHGRU_FMA_PER_STEP = 128


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured", j
    except Exception:
        return 6650.0, "fallback", {}


def measure_pipe_peak(pr, pipe, device, local, target_ms=150.0):
    """Measured peak of one functional-unit pipe on this GPU: the library's
    throughput probe (ex2 + rcp for the special-function pipe, fp32 FMA)
    timed with CUDA events over about `target_ms`, with the SM clock sampled
    meanwhile.  Returns the rate per SM per clock, so that a kernel timed at
    another clock is compared with the peak at its own clock."""
    import torch

    sink = torch.zeros(1, device=device)
    stream = torch.cuda.current_stream(device)
    iters = 64
    for _ in range(2):                      # warm-up
        pr.probe_rate(pipe, iters, sink)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    pr.probe_rate(pipe, iters, sink)
    e1.record(stream)
    torch.cuda.synchronize()
    one = max(e0.elapsed_time(e1), 1e-3)
    iters = int(max(64, min(1 << 20, iters * 2.0 / one)))    # ~2 ms per launch
    n = int(max(4, target_ms / 2.0))
    pr.probe_rate(pipe, iters, sink)
    torch.cuda.synchronize()
    with ClockSampler(local, period_s=0.002) as clk:
        e0.record(stream)
        ops = sum(pr.probe_rate(pipe, iters, sink) for _ in range(n))
        e1.record(stream)
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    c = clk.summary()
    nsm = torch.cuda.get_device_properties(device).multi_processor_count
    mhz = c.get("sm_mhz") or 1965.0
    rate = ops / (ms * 1e-3)
    return {"ops_per_s": rate, "per_sm_per_clk": rate / (nsm * mhz * 1e6), "sm_mhz": mhz,
            "sms": nsm, "ms": ms, "launches": n, "clock_reasons": c.get("reasons"),
            "clock_source": c.get("source")}


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    """Samples the SM clock and the throttle reasons every few ms through NVML
    (read-only queries) while the timed region runs."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, gpu_index, period_s=0.005):
        self.gpu = gpu_index
        self.period = period_s
        self.samples = []
        self.smax = None
        self._stop = threading.Event()
        self._nvml = None

    def __enter__(self):
        try:
            import pynvml

            pynvml.nvmlInit()
            self._nvml = pynvml
            uuid = None
            try:
                import torch

                uuid = str(torch.cuda.get_device_properties(self.gpu).uuid)
            except Exception:
                pass
            h = None
            if uuid:
                try:
                    h = pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid).encode())
                except Exception:
                    h = None
            self.h = h if h is not None else pynvml.nvmlDeviceGetHandleByIndex(self.gpu)
            self.smax = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self._sample()
            self.t = threading.Thread(target=self._loop, daemon=True)
            self.t.start()
        except Exception:
            self._nvml = None
        return self

    def _sample(self):
        p = self._nvml
        sm = p.nvmlDeviceGetClockInfo(self.h, p.NVML_CLOCK_SM)
        try:
            r = p.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            r = p.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
        self.samples.append((sm, int(r)))

    def _loop(self):
        # the first sample is taken by __enter__; the thread waits a period
        # before each further one, so its start does not delay the first launch
        while not self._stop.wait(self.period):
            try:
                self._sample()
            except Exception:
                break

    def __exit__(self, *exc):
        self._stop.set()
        if self._nvml is not None:
            try:
                self.t.join(timeout=2)
                self._sample()
            except Exception:
                pass

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        reasons = set()
        for _, r in self.samples:
            for name, bit in self.REASONS.items():
                if r & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(s for s, _ in self.samples), "sm_max_mhz": self.smax,
                "reasons": sorted(reasons), "samples": len(self.samples), "source": "nvml"}


# ---------------------------------------------------------------------------
# distributed plumbing (weak scaling: one independent batch per rank)
# ---------------------------------------------------------------------------
def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def maybe_init_pg(world, backend):
    import torch.distributed as dist
    from datetime import timedelta

    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=timedelta(seconds=120))
    return dist


def max_over_ranks(val, world, device):
    if world == 1:
        return val
    import torch
    import torch.distributed as dist

    t = torch.tensor([val], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def aggregate(ms_local, world, units_per_rank, device):
    """Whole-job throughput under weak scaling: every rank processed
    `units_per_rank` channel-steps per step; the step time is the slowest rank's."""
    ms = max_over_ranks(ms_local, world, device)
    return ms, world * units_per_rank / (ms * 1e-3)


# ---------------------------------------------------------------------------
# sweep accounting (mirrors the kernel's schedule: m_first then m_next per sweep)
# ---------------------------------------------------------------------------
def evaluated_iterations(passes, max_iters, m_first=4, m_next=2):
    k0, total = 0, 0
    for q in range(passes):
        m = m_first if q == 0 else m_next
        m = min(m, max_iters + 1 - k0)
        total += m
        k0 += m
    return total


def algorithmic_bytes(op, bf16, B, L, D, passes=1):
    """Bytes one launch must move.  Solves: each sweep reads P once, reads the
    iterate (not in the first sweep: h^0 = 0) and writes the new iterate.
    Scans: read A and b, write the state once."""
    N = B * L * D
    if op == "scan_diag":
        return 12 * N
    if op == "scan_block2":
        return 32 * N
    if op in ("proj", "proj_solve"):  # handled by projection_bytes (depends on K and G)
        raise ValueError("use projection_bytes for the input projection")
    if op == "mhgru":     # one evaluation: read P, the iterate, write the iterate
        return N * (12 + 4 + 4) * passes
    if op == "gru_bwd":   # read P, h_{t-1}, dl/dh; write dP
        return N * (3 * (2 if bf16 else 4) + 4 + 4 + 12)
    if op == "lstm_bwd":  # read P, (c, h)_{t-1}, dl/dc, dl/dh; write dP
        return N * (4 * (2 if bf16 else 4) + 8 + 8 + 16)
    G = 3 if op == "gru" else 4
    ns = 1 if op == "gru" else 2
    pbytes = G * (2 if bf16 else 4)
    first = pbytes + 4 * ns
    later = pbytes + 8 * ns
    return N * (first + later * (passes - 1))


def projection_bytes(M, N, K, out_bf16):
    """Bytes the projection must move: x and W once (bf16), the bias, P once."""
    return 2 * M * K + 2 * N * K + 4 * N + (2 if out_bf16 else 4) * M * N


def kernel_source_digest():
    """sha256 of the CUDA sources: ties a recorded ncu traffic figure to the
    kernel it was measured on."""
    import hashlib

    hsh = hashlib.sha256()
    csrc = os.path.join(ROOT, "nonlinear_rnn_solve_newton_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, name), "rb") as f:
            hsh.update(name.encode() + b"\0" + f.read())
    return hsh.hexdigest()


def recorded_traffic(workload):
    """DRAM bytes per launch measured by ncu (profiles/traffic.json), or None
    if no capture exists or the kernels changed since it was taken."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f)
    except Exception:
        return None, "no capture recorded"
    k = rec.get("kernels", {}).get(workload)
    if not k:
        return None, "no capture for this workload"
    # each capture carries the digest of the sources it was taken on
    if k.get("source_sha256", rec.get("source_sha256")) != kernel_source_digest():
        return None, "kernels changed since the capture"
    # a capture of a shorter sequence, scaled to the full launch by the
    # channel-steps it processes (the walker's traffic grows with L)
    scale = float(k.get("scale", 1))
    src = "ncu " + k.get("capture", "")
    if scale != 1:
        src += f", x {scale:g} to the full length"
    return int(round(k["dram_bytes_per_launch"] * scale)), src


# ---------------------------------------------------------------------------
# workloads: device inputs, one step, host copies for the end-to-end leg
# ---------------------------------------------------------------------------
class Case:
    def __init__(self, name, rank, device, seq_len=None, proj_k=None):
        import torch

        import nonlinear_rnn_solve_newton_b200 as pr

        self.pr = pr
        self.name = name
        w = dict(inputs.WORKLOADS[name])
        base_seed = w["seed"]
        if seq_len is not None:
            # the sequence-length sweep: the same draws as tests.inputs.workload_inputs(name, L)
            w["L"] = int(seq_len)
            base_seed = [w["seed"], int(seq_len)]
        if proj_k is not None and "K" in w:
            # another input width for the projection workloads (its own draws)
            w["K"] = int(proj_k)
            base_seed = [base_seed, 7000 + int(proj_k)] if not isinstance(base_seed, list) else \
                base_seed + [7000 + int(proj_k)]
        self.w = w
        self.op, self.B, self.L, self.D, self.bf16 = w["op"], w["B"], w["L"], w["D"], w["bf16"]
        self.N = self.B * self.L * self.D
        self.device = device
        self.tol, self.max_iters = 1e-4, 32
        seed = base_seed if rank == 0 else [base_seed, 1000 + rank] if not isinstance(
            base_seed, list) else base_seed + [1000 + rank]
        B, L, D = self.B, self.L, self.D
        self.out_dtype = None
        if self.op == "proj":
            # x [B, L, K] -> P [B, L, G, D]: M = B * L rows, N = G * D features
            self.K, self.G = w["K"], w["G"]
            M, Nf = B * L, w["G"] * D
            x = inputs.projection_inputs(M, Nf, self.K, seed)
            x["G"] = self.G
            self.host = {
                "x": torch.from_numpy(x["x_bits"].view(np.int16)).view(torch.bfloat16).view(
                    B, L, self.K),
                "W": torch.from_numpy(x["W_bits"].view(np.int16)).view(torch.bfloat16),
                "bias": torch.from_numpy(x["bias"])}
            self.out_dtype = torch.bfloat16 if self.bf16 else torch.float32
            self.out_shapes = [(B, L, Nf)]
        elif self.op == "proj_solve":
            # x [B, L, K] and W [3 D, K] (bf16) -> the ParaGRU solve, P kept on chip
            self.K, self.G = w["K"], 3
            x = inputs.projected_gru_inputs(B, L, D, self.K, seed)
            self.host = {
                "x": torch.from_numpy(x["x_bits"].view(np.int16)).view(torch.bfloat16),
                "W": torch.from_numpy(x["W_bits"].view(np.int16)).view(torch.bfloat16),
                "bias": torch.from_numpy(x["bias"]), "a": torch.from_numpy(x["a"]),
                "h0": torch.from_numpy(x["h0"])}
            self.out_shapes = [(B, L, D)]
        elif self.op in ("gru_bwd", "lstm_bwd"):
            # the backward pass differentiates the forward solution: solve once here
            cell = self.op[:-4]
            x = (inputs.gru_inputs if cell == "gru" else inputs.lstm_inputs)(B, L, D, seed,
                                                                               self.bf16)
            P = torch.from_numpy(x["P"])
            self.host = {"P": P, "a": torch.from_numpy(x["a"]), "h0": torch.from_numpy(x["h0"])}
            grads = inputs.upstream_gradients(B, L, D, w["seed"], 2 if cell == "lstm" else 1)
            self.host["gh"] = torch.from_numpy(grads[0])
            if cell == "lstm":
                self.host["c0"] = torch.from_numpy(x["c0"])
                self.host["gc"] = torch.from_numpy(grads[1])
            dv = {k: v.to(device) for k, v in self.host.items()}
            if cell == "gru":
                hs, info = pr.solve_gru(dv["P"], dv["a"], dv["h0"])
                self.host["h"] = hs.cpu()
            else:
                cs_, hs, info = pr.solve_lstm(dv["P"], dv["a"], dv["c0"], dv["h0"])
                self.host["c"] = cs_.cpu()
                self.host["h"] = hs.cpu()
            G = 3 if cell == "gru" else 4
            self.out_shapes = [(B, L, G, D), (G, D), (B, D)] + ([(B, D)] if cell == "lstm" else [])
        elif self.op == "mhgru":
            x = inputs.mhgru_inputs(B, L, D // 8, seed)
            self.host = {"P": torch.from_numpy(x["P"]), "U": torch.from_numpy(x["U"])}
            self.out_shapes = [(B, L, D)]
        elif self.op in ("gru", "lstm"):
            x = (inputs.gru_inputs if self.op == "gru" else inputs.lstm_inputs)(B, L, D, seed,
                                                                                  self.bf16)
            if self.bf16:
                P = torch.from_numpy(x["P_bits"].view(np.int16)).view(torch.bfloat16)
            else:
                P = torch.from_numpy(x["P"])
            self.host = {"P": P, "a": torch.from_numpy(x["a"]), "h0": torch.from_numpy(x["h0"])}
            if self.op == "lstm":
                self.host["c0"] = torch.from_numpy(x["c0"])
            self.out_shapes = [(B, L, D)] * (2 if self.op == "lstm" else 1)
        elif self.op == "scan_diag":
            x = inputs.scan_diag_inputs(B, L, D, seed)
            self.host = {k: torch.from_numpy(v) for k, v in x.items()}
            self.out_shapes = [(B, L, D)]
        else:
            x = inputs.scan_block2_inputs(B, L, D, seed)
            self.host = {k: torch.from_numpy(v) for k, v in x.items()}
            self.out_shapes = [(B, L, D, 2)]
        self.x = x
        self.dev = {k: v.to(device) for k, v in self.host.items()}
        odt = self.out_dtype or torch.float32
        self.outs = [torch.empty(sh, dtype=odt, device=device) for sh in self.out_shapes]
        self.info_t = torch.empty(pr.INFO_BYTES // 4, dtype=torch.int32, device=device)

    def run(self, d, outs):
        pr, op = self.pr, self.op
        if op == "gru":
            pr.solve_gru(d["P"], d["a"], d["h0"], self.tol, self.max_iters, out=outs[0],
                         info=self.info_t)
        elif op == "lstm":
            pr.solve_lstm(d["P"], d["a"], d["c0"], d["h0"], self.tol, self.max_iters,
                          out=(outs[0], outs[1]), info=self.info_t)
        elif op == "mhgru":
            pr.solve_mhgru(d["P"], d["U"], None, self.tol, self.max_iters, out=outs[0],
                           info=self.info_t)
        elif op == "proj":
            pr.input_projection(d["x"], d["W"], d["bias"], out=outs[0], out_dtype=self.out_dtype)
        elif op == "proj_solve":
            pr.solve_gru_projected(d["x"], d["W"], d["bias"], d["a"], d["h0"], self.tol,
                                   self.max_iters, out=outs[0], info=self.info_t)
        elif op == "gru_bwd":
            pr.solve_gru_backward(d["P"], d["a"], d["h"], d["gh"], d["h0"],
                                  out=(outs[0], outs[1], outs[2]))
        elif op == "lstm_bwd":
            pr.solve_lstm_backward(d["P"], d["a"], d["c"], d["h"], d["gc"], d["gh"], d["c0"],
                                   d["h0"], out=(outs[0], outs[1], outs[2], outs[3]))
        elif op == "scan_diag":
            pr.scan_diag(d["A"], d["b"], d["h0"], out=outs[0])
        else:
            pr.scan_block2(d["A"], d["b"], d["x0"], out=outs[0])

    def step(self):
        self.run(self.dev, self.outs)

    def solve_info(self):
        if self.op in ("gru", "lstm", "mhgru", "proj_solve"):
            return self.pr.SolveInfo(self.info_t)
        return None


def workload_name(name, B, L, D, K=None, G=None):
    """The `config.workload` string of a workload (the same in both arms)."""
    wl = {"gru_l": "ParaGRU Newton solve fp32",
          "lm": "ParaGRU Newton solve, bf16 P, fp32 state",
          "deer": "ParaGRU Newton solve fp32 (DEER shape)",
          "gru_s": "ParaGRU Newton solve fp32 (small)",
          "lstm": "ParaLSTM Newton solve fp32",
          "scan": "diagonal affine scan fp32",
          "scan_lm": "diagonal affine scan fp32 (LM width)",
          "block2": "2x2 block affine scan fp32",
          "gru_bwd": "ParaGRU backward pass fp32",
          "lstm_bwd": "ParaLSTM backward pass fp32",
          "mhgru": "multi-head GRU Newton solve fp32, dense 8x8 recurrence blocks",
          "proj": "input projection x W^T + bias, bf16 in, fp32 out (tcgen05)",
          "proj_lm": "input projection x W^T + bias, bf16 in, bf16 out (tcgen05)",
          "proj_solve": "ParaGRU layer from its inputs: projection x W^T + bias (tcgen05, "
                        "bf16 in, fp32 P kept on chip) fused with the Newton solve",
          }[name]
    out = f"{wl} B={B} L={L} D={D}"
    if K is not None:
        out += f" K={K} G={G} (M={B * L}, N={G * D})"
    return out


# the diagonal scan timed beside each solve workload (the scan half of the metric)
SCAN_LEG = {"lm": "scan_lm", "gru_l": "scan"}


def time_leg(name, K, W, warm_s, world, rank, device, stream):
    """A second workload of the run, timed like the main step: at least W
    untimed steps (and `warm_s` seconds), then K steps between CUDA events on
    the launching stream, max over ranks.  Returns (case, ms per step)."""
    import torch

    cs = Case(name, rank, device)
    n_w = 0
    t_w = time.perf_counter()
    while n_w < max(W, 3) or time.perf_counter() - t_w < warm_s:
        cs.step()
        n_w += 1
        if n_w % 8 == 0:
            torch.cuda.synchronize()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    barrier(world)
    torch.cuda.synchronize()
    ev[0].record(stream)
    for _ in range(K):
        cs.step()
    ev[1].record(stream)
    torch.cuda.synchronize()
    return cs, max_over_ranks(ev[0].elapsed_time(ev[1]) / K, world, device)


def scan_summary(sc, ms, world, hbm_peak, peak_kind):
    """The scan leg's line: its 12 algorithmic bytes per channel-step against
    the HBM copy bandwidth (measured, else the fallback; `hbm_peak_kind` says
    which) and against 8 TB/s."""
    sbytes = algorithmic_bytes("scan_diag", False, sc.B, sc.L, sc.D)
    sgbs = sbytes / (ms * 1e-3) / 1e9
    st, ssrc = recorded_traffic(sc.name)
    return {"workload": workload_name(sc.name, sc.B, sc.L, sc.D), "ms": ms,
            "channel_steps_per_s": world * sc.N / (ms * 1e-3), "achieved_gbs": sgbs,
            "algorithmic_bytes": sbytes, "frac_of_hbm_peak": sgbs / hbm_peak,
            "hbm_peak_gbs": hbm_peak, "hbm_peak_kind": peak_kind,
            "frac_of_8tbs": sgbs / 8000.0, "traffic": st, "traffic_source": ssrc}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def run_ours(args, world, rank, local):
    import torch

    import nonlinear_rnn_solve_newton_b200 as pr

    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    maybe_init_pg(world, "nccl")
    pr.load()
    cs = Case(args.workload, rank, device, args.seq_len, args.proj_k)
    op, B, L, D, bf16, N = cs.op, cs.B, cs.L, cs.D, cs.bf16, cs.N
    stream = torch.cuda.current_stream()

    # Warm-up: W untimed steps (at least 3), reported as "warmup".  Then more
    # untimed steps until the GPU has run the workload for --warmup-seconds, so
    # that clocks and memory have settled; those are reported separately as
    # "warmup_settle" (they only lengthen the untimed part of the run).
    W = 0
    while W < max(args.warmup, 3):
        cs.step()
        W += 1
    torch.cuda.synchronize()
    settle = 0
    t_w = time.perf_counter()
    while time.perf_counter() - t_w < args.warmup_seconds:
        cs.step()
        settle += 1
        if settle % 8 == 0:
            torch.cuda.synchronize()
    torch.cuda.synchronize()
    info = cs.solve_info()
    if info is not None and (info.status != 0 or not info.converged):
        raise SystemExit(f"solve did not converge: {info.as_dict()}")
    iters = info.iterations if info else None
    passes = info.passes if info else 1

    # ---- optional: the step as a CUDA graph (removes the per-call host cost
    # that dominates latency-bound workloads; the graph holds the same launches)
    graph = None
    # (default: the small and the short-sequence workloads, where host-side call
    # cost is a visible part of a step)
    use_graph = (args.graph if args.graph is not None
                 else args.workload == "gru_s" or (args.seq_len is not None and args.seq_len <= 1024))
    if use_graph:
        gs = torch.cuda.Stream(device)
        gs.wait_stream(stream)
        with torch.cuda.stream(gs):
            cs.step()
        stream.wait_stream(gs)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=gs):
            cs.step()
        torch.cuda.synchronize()
        for _ in range(3):
            graph.replay()
        torch.cuda.synchronize()
    run_step = graph.replay if graph is not None else cs.step

    # One untimed pass shaped like the timed loop (back-to-back steps, events on
    # the stream), counted in warmup_settle.  The first such pass of a process
    # ran its first step ~0.07 ms slower than later ones on B200.
    pre = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    pre[0].record(stream)
    for i in range(3):
        run_step()
        pre[i + 1].record(stream)
        settle += 1
    torch.cuda.synchronize()

    # ---- timed region: exactly K steps ---------------------------------------
    K = args.steps
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(K + 1)]
    # The clock sampler (NVML queries, its thread) starts before the bracket,
    # so its start-up is not timed.
    with ClockSampler(local) as clk:
        barrier(world)
        torch.cuda.synchronize()
        evs[0].record(stream)
        for i in range(K):
            run_step()
            evs[i + 1].record(stream)
        torch.cuda.synchronize()
    barrier(world)
    per_step = [evs[i].elapsed_time(evs[i + 1]) for i in range(K)]
    ms_local = evs[0].elapsed_time(evs[K]) / K
    ms, value = aggregate(ms_local, world, N, device)
    clocks = clk.summary()

    # ---- roofline of the step's one kernel launch ----------------------------
    # Per-launch times are CUDA events around each call on the launching stream
    # (they also hold the ~2 us zeroing of the workspace control block).
    launch_ms = statistics.mean(per_step)
    hbm_peak, peak_kind, pk = peaks()
    if op == "proj":
        bytes_launch = projection_bytes(B * L, cs.G * D, cs.K, bf16)
    elif op == "proj_solve":
        # x and W once per sweep, the bias, the trajectory written once; no P
        bytes_launch = passes * (2 * B * L * cs.K + 2 * 3 * D * cs.K) + 4 * 3 * D + 4 * B * L * D
    else:
        bytes_launch = algorithmic_bytes(op, bf16, B, L, D, passes)
    achieved_gbs = bytes_launch / (launch_ms * 1e-3) / 1e9
    hbm_frac = achieved_gbs / hbm_peak
    traffic, traffic_src = recorded_traffic(args.workload)
    mufu_probe = None
    hbm = {"bound": "hbm", "achieved": achieved_gbs, "peak": hbm_peak, "unit": "GB/s",
           "frac": hbm_frac, "traffic": traffic, "peak_kind": peak_kind,
           "algorithmic_bytes_per_launch": bytes_launch}
    if op in ("gru", "lstm", "gru_bwd", "lstm_bwd"):
        if op in ("gru", "lstm"):
            ev_iters = evaluated_iterations(passes, cs.max_iters,
                                            m_first=5 if op == "lstm" else 4)
        else:
            ev_iters = 1  # the backward evaluates each step once
        mufu_ops = N * ev_iters * MUFU_PER_STEP[op[:4].rstrip("_")]
        sm_mhz = clocks.get("sm_mhz") or pk.get("sm_max_mhz", 1965.0)
        probe = mufu_probe = measure_pipe_peak(pr, pr.PROBE_MUFU, device, local)
        mufu_peak = probe["per_sm_per_clk"] * probe["sms"] * sm_mhz * 1e6
        alu = {"bound": "alu", "achieved": mufu_ops / (launch_ms * 1e-3) / 1e12,
               "peak": mufu_peak / 1e12, "unit": "Tops/s (MUFU ex2+rcp)",
               "frac": mufu_ops / (launch_ms * 1e-3) / mufu_peak, "traffic": traffic,
               "peak_kind": ("measured: ex2+rcp throughput probe, %.2f ops per SM per clock "
                             "at %.0f MHz, scaled to the timed region's SM clock"
                             % (probe["per_sm_per_clk"], probe["sm_mhz"])),
               "peak_probe": probe, "mufu_ops_per_launch": mufu_ops}
        if alu["frac"] >= hbm_frac:
            roofline = dict(alu)
            roofline["hbm"] = {k: hbm[k] for k in ("achieved", "peak", "peak_kind", "unit", "frac",
                                                    "algorithmic_bytes_per_launch")}
        else:
            roofline = dict(hbm)
            roofline["alu"] = {k: alu[k] for k in ("achieved", "peak", "unit", "frac")}
    elif op == "mhgru":
        ev_iters = (iters or 0) + 1
        sm_mhz = clocks.get("sm_mhz") or pk.get("sm_max_mhz", 1965.0)
        flops = 2.0 * N * ev_iters * MHGRU_FMA_PER_STEP
        probe = measure_pipe_peak(pr, pr.PROBE_FMA, device, local)
        fpeak = probe["per_sm_per_clk"] * probe["sms"] * 2 * sm_mhz * 1e6 / 1e12
        ach = flops / (launch_ms * 1e-3) / 1e12
        roofline = {"bound": "alu", "achieved": ach, "peak": fpeak,
                    "unit": "TFLOP/s (fp32 FMA, CUDA cores)", "frac": ach / fpeak,
                    "traffic": traffic, "flops_per_launch": flops,
                    "peak_kind": ("measured: fp32 FMA throughput probe, %.1f FMA per SM per "
                                  "clock at %.0f MHz, scaled to the timed region's SM clock"
                                  % (probe["per_sm_per_clk"], probe["sm_mhz"])),
                    "peak_probe": probe,
                    "hbm": {"achieved": achieved_gbs, "peak": hbm_peak, "peak_kind": peak_kind, "unit": "GB/s",
                            "frac": hbm_frac}}
    elif op == "proj_solve":
        ev_iters = evaluated_iterations(passes, cs.max_iters)
        flops = 2.0 * (B * L) * (3 * D) * cs.K * passes
        tf_peak = pk.get("bf16_tflops")
        tf_kind = "measured burst (cuBLAS bf16 GEMM, MEASURED_PEAKS)"
        if not tf_peak:
            tf_peak, tf_kind = 1590.0, "fallback"
        tflops = flops / (launch_ms * 1e-3) / 1e12
        sm_mhz = clocks.get("sm_mhz") or pk.get("sm_max_mhz", 1965.0)
        probe = mufu_probe = measure_pipe_peak(pr, pr.PROBE_MUFU, device, local)
        mufu_ops = N * ev_iters * MUFU_PER_STEP["gru"]
        mufu_peak = probe["per_sm_per_clk"] * probe["sms"] * sm_mhz * 1e6
        roofline = {"bound": "tensor", "achieved": tflops, "peak": tf_peak, "unit": "TFLOP/s",
                    "frac": tflops / tf_peak, "traffic": traffic, "peak_kind": tf_kind,
                    "flops_per_launch": flops,
                    "alu": {"achieved": mufu_ops / (launch_ms * 1e-3) / 1e12,
                            "peak": mufu_peak / 1e12, "unit": "Tops/s (MUFU ex2+rcp)",
                            "frac": mufu_ops / (launch_ms * 1e-3) / mufu_peak,
                            "peak_kind": "measured: ex2+rcp throughput probe"},
                    "hbm": {"achieved": achieved_gbs, "peak": hbm_peak, "peak_kind": peak_kind, "unit": "GB/s",
                            "frac": hbm_frac, "algorithmic_bytes_per_launch": bytes_launch}}
    elif op == "proj":
        ev_iters = None
        flops = 2.0 * (B * L) * (cs.G * D) * cs.K
        tf_peak = pk.get("bf16_tflops")
        tf_kind = "measured burst (cuBLAS bf16 GEMM, MEASURED_PEAKS)"
        if not tf_peak:
            tf_peak, tf_kind = 1590.0, "fallback"
        tflops = flops / (launch_ms * 1e-3) / 1e12
        roofline = {"bound": "tensor", "achieved": tflops, "peak": tf_peak, "unit": "TFLOP/s",
                    "frac": tflops / tf_peak, "traffic": traffic, "peak_kind": tf_kind,
                    "flops_per_launch": flops,
                    "hbm": {"achieved": achieved_gbs, "peak": hbm_peak, "peak_kind": peak_kind, "unit": "GB/s",
                            "frac": hbm_frac, "algorithmic_bytes_per_launch": bytes_launch}}
    else:
        ev_iters = None
        roofline = dict(hbm)
    roofline["kernel"] = {"gru": "pararnn Newton kernel (GRU)", "lstm":
                          "pararnn Newton kernel (LSTM)", "scan_diag": "pararnn scan (diagonal)",
                          "scan_block2": "pararnn scan (2x2)",
                          "gru_bwd": "pararnn backward kernel (GRU)",
                          "lstm_bwd": "pararnn backward kernel (LSTM)",
                          "proj": "pararnn input projection (tcgen05)",
                          "proj_solve": "pararnn projection fused with the GRU Newton walk "
                                        "(tcgen05 + CUDA cores)",
                          "mhgru": "pararnn multi-head GRU Newton kernel (8x8 blocks)"}[op]
    roofline["launch_ms"] = launch_ms
    roofline["traffic_source"] = traffic_src

    # ---- the diagonal scan at the same width (the scan half of the metric) --
    scan = None
    scan_name = SCAN_LEG.get(args.workload)
    if scan_name and not args.no_scan:
        sc, sms = time_leg(scan_name, K, W, args.warmup_seconds, world, rank, device, stream)
        scan = scan_summary(sc, sms, world, hbm_peak, peak_kind)
        del sc

    # ---- the fused layer against the unfused pair (P through HBM) ------------
    unfused = None
    if op == "proj_solve" and not args.no_extra:
        d = cs.dev
        Pbuf = torch.empty((B, L, 3 * D), dtype=torch.bfloat16, device=device)
        hbuf = torch.empty((B, L, D), dtype=torch.float32, device=device)

        def pair():
            pr.input_projection(d["x"], d["W"], d["bias"], out=Pbuf, out_dtype=torch.bfloat16)
            pr.solve_gru(Pbuf.view(B, L, 3, D), d["a"], d["h0"], cs.tol, cs.max_iters,
                         out=hbuf, info=cs.info_t)
        for _ in range(max(W, 3)):
            pair()
        torch.cuda.synchronize()
        pev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        barrier(world)
        pev[0].record(stream)
        for _ in range(K):
            pair()
        pev[1].record(stream)
        torch.cuda.synchronize()
        pms = max_over_ranks(pev[0].elapsed_time(pev[1]) / K, world, device)
        unfused = {"what": "pararnn_input_projection (bf16 P to HBM) then pararnn_solve_gru "
                           "(bf16 P read back), same inputs", "ms": pms,
                   "fused_speedup": pms / ms,
                   "max_abs_diff_vs_fused": float(torch.max(torch.abs(hbuf - cs.outs[0])).item())}
        del Pbuf, hbuf

    # ---- extra keys: the fp32 solve and scan at B=8, L=4096, D=1024 ----------
    extra = None
    if args.workload == "lm" and not args.no_extra:
        g, gms = time_leg("gru_l", K, W, args.warmup_seconds, world, rank, device, stream)
        ginfo = g.solve_info()
        gpasses = ginfo.passes
        gev = evaluated_iterations(gpasses, g.max_iters)
        gmufu = g.N * gev * MUFU_PER_STEP["gru"]
        gbytes = algorithmic_bytes("gru", False, g.B, g.L, g.D, gpasses)
        gsm = clocks.get("sm_mhz") or pk.get("sm_max_mhz", 1965.0)
        if mufu_probe is None:
            mufu_probe = measure_pipe_peak(pr, pr.PROBE_MUFU, device, local)
        gpeak = mufu_probe["per_sm_per_clk"] * mufu_probe["sms"] * gsm * 1e6
        gtr, gtsrc = recorded_traffic("gru_l")
        extra = {"workload": workload_name("gru_l", g.B, g.L, g.D), "ms": gms,
                 "channel_steps_per_s": world * g.N / (gms * 1e-3),
                 "newton_iterations": ginfo.iterations, "sweeps": gpasses,
                 "evaluated_iterations": gev,
                 "mufu_frac": gmufu / (gms * 1e-3) / gpeak,
                 "hbm_gbs": gbytes / (gms * 1e-3) / 1e9,
                 "hbm_frac": gbytes / (gms * 1e-3) / 1e9 / hbm_peak,
                 "traffic": gtr, "traffic_source": gtsrc}
        del g
        sc, sms = time_leg("scan", K, W, args.warmup_seconds, world, rank, device, stream)
        extra["scan"] = scan_summary(sc, sms, world, hbm_peak, peak_kind)
        del sc

    # ---- context: sequential application on the same GPU ---------------------
    # (ParaRNN's abstract measures its speedup against naive sequential
    # application: one launch per time step.  Also timed: the one-thread-per-
    # channel rollout, whose time is L x the cell's dependency chain.)
    sequential = None
    if op == "mhgru" and not args.no_sequential:
        # the multi-head cell applied in order (8 lanes per head): the DEER
        # summary's caveat is that dense blocks make each Newton step O(n^3)
        try:
            d = cs.dev
            hroll = torch.empty((B, L, D), dtype=torch.float32, device=device)
            for _ in range(2):
                pr.rollout_mhgru(d["P"], d["U"], out=hroll)
            torch.cuda.synchronize()
            qev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
            Kq = max(1, min(K, 5))
            qev[0].record(stream)
            for _ in range(Kq):
                pr.rollout_mhgru(d["P"], d["U"], out=hroll)
            qev[1].record(stream)
            torch.cuda.synchronize()
            roll_ms = qev[0].elapsed_time(qev[1]) / Kq
            sequential = {"rollout_8_lanes_per_head_ms": roll_ms,
                          "newton_speedup_vs_rollout": roll_ms / ms}
            del hroll
        except Exception as e:  # context only; never fails the benchmark
            sequential = {"error": str(e)[:200]}
    if op in ("gru", "lstm") and not args.no_sequential:
        try:
            seq_fn = pr.rollout_gru if op == "gru" else pr.rollout_lstm
            d = cs.dev
            seq_args = (d["P"], d["a"], d["h0"]) if op == "gru" else (d["P"], d["a"], d["c0"],
                                                                      d["h0"])
            for _ in range(2):
                seq_fn(*seq_args)
            torch.cuda.synchronize()
            qev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
            Kq = max(1, min(K, 5))
            qev[0].record(stream)
            for _ in range(Kq):
                seq_fn(*seq_args)
            qev[1].record(stream)
            torch.cuda.synchronize()
            roll_ms = qev[0].elapsed_time(qev[1]) / Kq
            # naive loop: one decode-step launch per time step, over a bounded
            # number of steps, scaled to L
            nsteps = min(L, 2048)
            G = 3 if op == "gru" else 4
            Pt = d["P"][:, :nsteps].transpose(0, 1).contiguous()      # [n, B, G, D]
            hs = torch.empty((nsteps, B, D), dtype=torch.float32, device=device)
            cs_ = torch.empty_like(hs) if op == "lstm" else None

            def naive():
                prev_h = d["h0"]
                prev_c = d["c0"] if op == "lstm" else None
                for t in range(nsteps):
                    if op == "gru":
                        pr.step_gru(Pt[t], d["a"], prev_h, out=hs[t])
                    else:
                        pr.step_lstm(Pt[t], d["a"], prev_c, prev_h, out=(cs_[t], hs[t]))
                        prev_c = cs_[t]
                    prev_h = hs[t]
            naive()
            torch.cuda.synchronize()
            qev[0].record(stream)
            naive()
            qev[1].record(stream)
            torch.cuda.synchronize()
            naive_ms = qev[0].elapsed_time(qev[1]) * L / nsteps
            sequential = {"rollout_one_thread_per_channel_ms": roll_ms,
                          "naive_step_loop_ms": naive_ms,
                          "naive_step_loop_sample": f"{nsteps} of {L} steps, scaled",
                          "newton_speedup_vs_rollout": roll_ms / ms,
                          "newton_speedup_vs_naive_loop": naive_ms / ms}
            del Pt, hs, cs_
        except Exception as e:  # context only; never fails the benchmark
            sequential = {"error": str(e)[:200]}

    # ---- end to end through the public API with pinned host buffers ---------
    # Every step copies its inputs host -> device, solves through the public
    # binding and copies the result device -> host.  Three streams and two
    # device slots let step i's result copy overlap step i+1's input copy
    # (PCIe is full duplex); the timed region spans all copies of all steps.
    e2e = None
    if not args.no_e2e:
        pin = {k: v.pin_memory() for k, v in cs.host.items()}
        odt = cs.out_dtype or torch.float32
        outs_pin = [[torch.empty(sh, dtype=odt).pin_memory() for sh in cs.out_shapes]
                    for _ in range(2)]
        dev_in = [{k: torch.empty_like(v, device=device) for k, v in pin.items()}
                  for _ in range(2)]
        dev_out = [[torch.empty(sh, dtype=odt, device=device) for sh in cs.out_shapes]
                   for _ in range(2)]
        s_in, s_cmp, s_out = (torch.cuda.Stream(device) for _ in range(3))
        ev = {name: [torch.cuda.Event() for _ in range(2)]
              for name in ("in", "cmp", "out")}
        used = [False, False]

        def e2e_step(i):
            j = i % 2
            with torch.cuda.stream(s_in):
                if used[j]:
                    s_in.wait_event(ev["cmp"][j])       # the slot's inputs are consumed
                for k, v in pin.items():
                    dev_in[j][k].copy_(v, non_blocking=True)
                ev["in"][j].record(s_in)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(ev["in"][j])
                if used[j]:
                    s_cmp.wait_event(ev["out"][j])      # the slot's outputs are copied out
                cs.run(dev_in[j], dev_out[j])
                ev["cmp"][j].record(s_cmp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev["cmp"][j])
                for o_pin, o_dev in zip(outs_pin[j], dev_out[j]):
                    o_pin.copy_(o_dev, non_blocking=True)
                ev["out"][j].record(s_out)
            used[j] = True

        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize()
        Ke = min(K, 5)
        t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize()
        t_start.record(s_in)
        for i in range(Ke):
            e2e_step(i)
        s_in.wait_stream(s_out)
        s_in.wait_stream(s_cmp)
        t_end.record(s_in)
        torch.cuda.synchronize()
        ems = max_over_ranks(t_start.elapsed_time(t_end) / Ke, world, device)
        h2d = sum(v.numel() * v.element_size() for v in pin.values())
        d2h = sum(o.numel() * o.element_size() for o in outs_pin[0])
        e2e = {"value": world * N / (ems * 1e-3), "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": ems,
               "pipeline": "copy-in / solve / copy-out on three streams, two device slots"}
        del dev_in, dev_out

    # ---- the oracle on the host cores (rank 0, N = 1 only) -------------------
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_baseline(cs.x, op, B, L, D, budget_s=args.cpu_seconds)

    if rank == 0:
        kg = op in ("proj", "proj_solve")
        wlname = workload_name(args.workload, B, L, D, cs.K if kg else None,
                               cs.G if kg else None)
        cfg = {"workload": wlname, "B": B, "L": L, "D": D,
               "launch": "CUDA graph replay" if graph is not None else "direct calls",
               "parallelism": f"replicas x{world} (independent batches)",
               "l2": "inputs larger than L2 (%.0f MB per step), no flush needed" % (
                   sum(v.numel() * v.element_size() for v in cs.host.values()) / 1e6)}
        if op == "proj_solve":
            cfg.update({"K": cs.K})
        if op in ("gru", "lstm", "mhgru", "proj_solve"):
            cfg.update({"tol": cs.tol, "max_iters": cs.max_iters, "newton_iterations": iters,
                        "sweeps": passes, "evaluated_iterations": ev_iters})
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": W,
            "warmup_settle": {"steps": settle, "seconds": args.warmup_seconds,
                              "why": "extra untimed steps until the GPU has run the workload "
                                     "this long, so clocks and memory have settled"},
            "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": ("bf16-in/f32-acc" if op in ("proj", "proj_solve") else
                      "f32" if not bf16 else "bf16-in/f32"),
            "data": "synthetic (seeded numpy; see tests/inputs.py)",
            "config": cfg, "roofline": roofline, "clocks": clocks, "e2e": e2e,
            "gpu_launches": K, "scan": scan, "cpu_baseline": cpu,
            "sequential_gpu": sequential, "gru_l": extra, "unfused_pair": unfused,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


def cpu_baseline(x, op, B, L, D, budget_s=15.0):
    """The oracle's serial Newton (and its sequential rollout) on the host cores,
    on a bounded sample of the workload: the first batch rows, as many channels
    as fit the time budget (estimated from a short calibration run).  For the
    scans, the oracle's sequential scan over the whole workload."""
    import oracle

    oracle.build()
    cores = oracle.get_threads()
    if op == "proj":
        # rows of the projection (each row is L-independent work: N x K sums)
        Wd = x["W"]
        t0 = time.perf_counter()
        oracle.input_projection(x["x"][:8], Wd, x["bias"])
        per_row = max((time.perf_counter() - t0) / 8, 1e-6)
        nrows = int(max(8, min(x["x"].shape[0], budget_s / per_row)))
        t0 = time.perf_counter()
        oracle.input_projection(x["x"][:nrows], Wd, x["bias"])
        dt = time.perf_counter() - t0
        Nf = Wd.shape[0]
        return {"value": nrows * (Nf // x["G"]) / dt, "unit": UNIT, "cores": cores,
                "kind": "oracle",
                "sample": f"fp64 projection of {nrows} of {x['x'].shape[0]} rows "
                          f"(N={Nf}, K={Wd.shape[1]}; {dt:.1f} s)"}
    if op == "proj_solve":
        # one batch row, as many channels as fit the budget: the fp64 projection
        # of those channels' three gate rows, then the serial fp64 Newton solve
        Bx, Lx, Kx = x["x"].shape
        Dx = x["a"].shape[1]

        def sample(nd):
            rows = np.concatenate([np.arange(nd), Dx + np.arange(nd), 2 * Dx + np.arange(nd)])
            Pc = oracle.input_projection(x["x"][0], x["W"][rows], x["bias"][rows])
            Pc = Pc.reshape(1, Lx, 3, nd)
            return oracle.newton_gru(Pc, x["a"][:, :nd], tol=1e-4, max_iters=32)
        t0 = time.perf_counter()
        sample(4)
        per = max((time.perf_counter() - t0) / 4, 1e-6)
        nd = int(max(4, min(Dx, budget_s / per)))
        t0 = time.perf_counter()
        res = sample(nd)
        dt = time.perf_counter() - t0
        return {"value": Lx * nd / dt, "unit": UNIT, "cores": cores, "kind": "oracle",
                "sample": f"fp64 projection (K={Kx}) + serial fp64 Newton, B=1 x D={nd} x "
                          f"L={Lx} ({res.iterations} iterations, {dt:.1f} s)"}
    if op == "mhgru":
        # whole heads of one batch row, as many as fit the budget
        t0 = time.perf_counter()
        oracle.newton_mhgru(x["P"][:1, :, :, :8], x["U"][:, :1])
        per_head = max(time.perf_counter() - t0, 1e-6)
        nh = int(max(1, min(D // 8, budget_s / per_head)))
        t0 = time.perf_counter()
        res = oracle.newton_mhgru(x["P"][:1, :, :, :8 * nh], x["U"][:, :nh])
        dt = time.perf_counter() - t0
        return {"value": L * 8 * nh / dt, "unit": UNIT, "cores": cores, "kind": "oracle",
                "sample": f"serial fp64 Newton, B=1 x {nh} heads x L={L} "
                          f"({res.iterations} iterations, {dt:.1f} s)"}
    if op in ("gru_bwd", "lstm_bwd"):
        nb = 1
        nd = min(D, 256)
        Ps = x["P"][:nb, :, :, :nd]
        as_ = x["a"][:, :nd]
        t0 = time.perf_counter()
        if op == "gru_bwd":
            hh = oracle.rollout_gru(Ps, as_)
            oracle.backward_gru(Ps, as_, hh, hh)
        else:
            cc, hh = oracle.rollout_lstm(Ps, as_)
            oracle.backward_lstm(Ps, as_, cc, hh, cc, hh)
        dt = time.perf_counter() - t0
        return {"value": nb * L * nd / dt, "unit": UNIT, "cores": cores, "kind": "oracle",
                "sample": f"fp64 rollout + adjoint on B={nb} x D={nd} x L={L} ({dt:.1f} s)"}
    if op in ("scan_diag", "scan_block2"):
        fn = oracle.scan_diag if op == "scan_diag" else oracle.scan_block2
        args = (x["A"], x["b"], x["h0"] if op == "scan_diag" else x["x0"])
        t0 = time.perf_counter()
        fn(*args)
        dt = time.perf_counter() - t0
        return {"value": B * L * D / dt, "unit": UNIT, "cores": cores, "kind": "oracle",
                "sample": f"sequential fp64 scan over the whole workload ({dt:.1f} s)"}
    # calibrate on 64 channels
    nd = min(D, 64)
    Pc = x["P"][:1, :, :, :nd]
    ac = x["a"][:, :nd]
    t0 = time.perf_counter()
    if op == "gru":
        oracle.newton_gru(Pc, ac, tol=1e-4, max_iters=32)
    else:
        oracle.newton_lstm(Pc, ac, tol=1e-4, max_iters=32)
    dt = max(time.perf_counter() - t0, 1e-6)
    per_chan = dt / nd
    nchan = int(max(1, min(B * D, budget_s / per_chan)))
    nb = max(1, min(B, nchan // D)) if nchan >= D else 1
    ndd = D if nchan >= D else nchan
    Ps = x["P"][:nb, :, :, :ndd]
    as_ = x["a"][:, :ndd]
    t0 = time.perf_counter()
    if op == "gru":
        res = oracle.newton_gru(Ps, as_, tol=1e-4, max_iters=32)
    else:
        res = oracle.newton_lstm(Ps, as_, tol=1e-4, max_iters=32)
    dt = time.perf_counter() - t0
    steps = nb * L * ndd
    t1 = time.perf_counter()
    if op == "gru":
        oracle.rollout_gru(Ps, as_)
    else:
        oracle.rollout_lstm(Ps, as_)
    dtr = time.perf_counter() - t1
    # the same two programs on one host thread, on the first channels of the
    # sample (about 3 s of single-threaded work, estimated from the calibration)
    n1 = int(max(1, min(ndd, 3.0 / max(per_chan * cores, 1e-9))))
    P1, a1 = Ps[:1, :, :, :n1], as_[:, :n1]
    oracle.set_threads(1)
    try:
        t2 = time.perf_counter()
        if op == "gru":
            oracle.newton_gru(P1, a1, tol=1e-4, max_iters=32)
        else:
            oracle.newton_lstm(P1, a1, tol=1e-4, max_iters=32)
        dt1 = time.perf_counter() - t2
        t3 = time.perf_counter()
        if op == "gru":
            oracle.rollout_gru(P1, a1)
        else:
            oracle.rollout_lstm(P1, a1)
        dtr1 = time.perf_counter() - t3
    finally:
        oracle.set_threads(0)
    return {"value": steps / dt, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"serial fp64 Newton on B={nb} x D={ndd} channels x L={L} "
                      f"({steps} channel-steps, {res.iterations} iterations, {dt:.1f} s)",
            "rollout_channel_steps_per_s": steps / dtr,
            "single_thread": {"newton_channel_steps_per_s": n1 * L / dt1,
                              "rollout_channel_steps_per_s": n1 * L / dtr1,
                              "sample": f"{n1} channels x L={L} on one host thread"}}


# ---------------------------------------------------------------------------
# reference arm: the oracle, as it stands, on the host cores
# ---------------------------------------------------------------------------
def run_reference(args, world, rank, local):
    if rank != 0:
        return
    import oracle

    oracle.build()
    w = dict(inputs.WORKLOADS[args.workload])
    op, B, L, D, bf16 = w["op"], w["B"], w["L"], w["D"], w["bf16"]
    cores = oracle.get_threads()
    # each step: the oracle on one batch row's first channels (a bounded sample)
    nd = min(D, 256)
    if op in ("gru_bwd", "lstm_bwd"):
        cell = op[:-4]
        x = (inputs.gru_inputs if cell == "gru" else inputs.lstm_inputs)(B, L, D, w["seed"])
        Ps = np.ascontiguousarray(x["P"][:1, :, :, :nd])
        as_ = np.ascontiguousarray(x["a"][:, :nd])
        g = [v[:1, :, :nd] for v in inputs.upstream_gradients(B, L, D, w["seed"],
                                                              2 if cell == "lstm" else 1)]
        if cell == "gru":
            hh = oracle.rollout_gru(Ps, as_)

            def step():
                return oracle.backward_gru(Ps, as_, hh, g[0])
        else:
            cc, hh = oracle.rollout_lstm(Ps, as_)

            def step():
                return oracle.backward_lstm(Ps, as_, cc, hh, g[1], g[0])
        what = "adjoint (backward) recursion"
        x = None
    elif op == "mhgru":
        x = inputs.mhgru_inputs(B, L, D // 8, w["seed"])
        nd = min(D, 32)
        Ps = np.ascontiguousarray(x["P"][:1, :, :, :nd])
        Us = np.ascontiguousarray(x["U"][:, : nd // 8])

        def step():
            return oracle.newton_mhgru(Ps, Us)
        what = "serial fp64 Newton (8x8 blocks)"
    elif op == "proj_solve":
        K = w["K"]
        x = inputs.projected_gru_inputs(B, L, D, K, w["seed"])
        nd = min(D, 16)
        rows = np.concatenate([np.arange(nd), D + np.arange(nd), 2 * D + np.arange(nd)])
        xs, Ws, bs = x["x"][0], np.ascontiguousarray(x["W"][rows]), x["bias"][rows]
        as_ = np.ascontiguousarray(x["a"][:, :nd])

        def step():
            Pc = oracle.input_projection(xs, Ws, bs).reshape(1, L, 3, nd)
            return oracle.newton_gru(Pc, as_, tol=1e-4, max_iters=32)
        what = f"fp64 projection (K={K}) + serial fp64 Newton"
    elif op == "proj":
        Nf, K = w["G"] * D, w["K"]
        x = inputs.projection_inputs(B * L, Nf, K, w["seed"])
        nrows = max(1, min(B * L, int(2e8 // max(Nf * K, 1))))  # about 0.2 G multiply-adds
        xs = np.ascontiguousarray(x["x"][:nrows])

        def step():
            return oracle.input_projection(xs, x["W"], x["bias"])
        what = f"fp64 input projection ({nrows} rows x N={Nf} x K={K})"
    else:
        x = inputs.workload_inputs(args.workload)  # the same draws as the GPU arm, then sliced
    if op in ("gru_bwd", "lstm_bwd", "proj", "mhgru", "proj_solve"):
        pass
    elif op in ("gru", "lstm"):
        Ps = np.ascontiguousarray(x["P"][:1, :, :, :nd])
        as_ = np.ascontiguousarray(x["a"][:, :nd])
        fn = oracle.newton_gru if op == "gru" else oracle.newton_lstm

        def step():
            return fn(Ps, as_, tol=1e-4, max_iters=32)
        what = "serial fp64 Newton"
    else:
        if op == "scan_diag":
            sargs = (x["A"][:1, :, :nd], x["b"][:1, :, :nd], x["h0"][:1, :nd])
            fn = oracle.scan_diag
        else:
            sargs = (x["A"][:1, :, :nd], x["b"][:1, :, :nd], x["x0"][:1, :nd])
            fn = oracle.scan_block2

        def step():
            return fn(*sargs)
        what = "sequential fp64 scan"

    for _ in range(max(args.warmup, 1)):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / args.steps
    steps = nrows * D if op == "proj" else L * nd
    value = steps / dt
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": max(args.warmup, 1), "ms_per_step": dt * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded numpy)",
            "config": {"workload": workload_name(args.workload, B, L, D,
                                                 w.get("K") if op in ("proj", "proj_solve")
                                                 else None,
                                                 w.get("G") if op in ("proj", "proj_solve")
                                                 else None),
                       "B": B, "L": L, "D": D, "parallelism": "rank 0 only, host cores",
                       "sample": (f"oracle {what}" if op == "proj"
                                  else f"oracle {what} on B=1 x D={nd} x L={L} per step")},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": (what if op == "proj" else f"B=1, D={nd}, L={L} per step")},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="lm",
                    choices=["lm", "gru_l", "deer", "gru_s", "lstm", "scan", "scan_lm", "block2",
                             "gru_bwd", "lstm_bwd", "proj", "proj_lm", "proj_solve", "mhgru"])
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu", action="store_true", help="skip the oracle CPU baseline")
    ap.add_argument("--no-scan", action="store_true", help="skip the scan leg (lm, gru_l)")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the extra keys of the lm workload (solve and scan at "
                         "B=8 L=4096 D=1024)")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer leg")
    ap.add_argument("--no-sequential", action="store_true",
                    help="skip the sequential-application context timings")
    ap.add_argument("--proj-k", type=int, default=None,
                    help="input width K of the projection workloads (proj, proj_lm, proj_solve)")
    ap.add_argument("--seq-len", type=int, default=None,
                    help="override L (the sequence-length sweep, e.g. 64 .. 16384 for gru_l)")
    ap.add_argument("--graph", dest="graph", action="store_true", default=None,
                    help="time the step as CUDA graph replays (default for gru_s)")
    ap.add_argument("--no-graph", dest="graph", action="store_false")
    ap.add_argument("--warmup-seconds", type=float, default=0.5,
                    help="keep warming up until this much time has passed (after W steps)")
    args = ap.parse_args()
    world, rank, local = dist_setup()
    if args.impl == "reference":
        run_reference(args, world, rank, local)
    else:
        run_ours(args, world, rank, local)


if __name__ == "__main__":
    main()
