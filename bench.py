"""Throughput of the Mamba-3 scan on B200 (tokens/s, B*T per second, all heads).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config I] [--impl ours|reference]

A step is one pass of the whole hot path over one batch of synthetic input:
for the chunked workloads one ``m3_siso_chunked_fwd`` / ``m3_mimo_chunked_fwd``
call (discretization, rotation and scan fused), for the decode workload one
``m3_step_decode`` over every (batch, head) lane.  The default workload is
the SISO 434M-layer shape (batch 8, seqlen 2048, 16 heads, headdim 64,
dState 128, chunk 64, bf16).

For N > 1 (torchrun) every rank runs an independent replica of the workload on
its own GPU: the (batch, head) lanes are independent, there is no exchange
step and no collective on the data path (weak scaling); rank 0 prints the
whole-job value = units of all ranks / max-over-ranks device time.

``--impl reference`` times the fp64 CPU oracle (the only reference this path
has) on the host cores, on a bounded sample of the same workload per step.
"""
import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from state_space_lm_b200 import inputs as gen  # noqa: E402

METRIC = "Mamba-3 scan tokens/s (B·T) at H=16 and % of tensor/HBM roofline, 1×B200"
UNIT = "tokens/s"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def launch_plan(gpus, env):
    """How a run asked for ``--gpus N`` proceeds, given the environment.

    Returns ("run", world) to run here as one rank of ``world``,
    ("relaunch", N) when N > 1 was asked without torchrun (the script starts
    itself again under torchrun with N ranks), or ("error", message) when
    torchrun's WORLD_SIZE disagrees with --gpus."""
    if gpus < 1:
        return "error", "--gpus must be >= 1 (got %d)" % gpus
    if "WORLD_SIZE" not in env:
        return ("relaunch", gpus) if gpus > 1 else ("run", 1)
    world = int(env["WORLD_SIZE"])
    if world != gpus:
        return "error", "--gpus %d but WORLD_SIZE=%d: launch %d ranks, or pass --gpus %d" % (
            gpus, world, gpus, world)
    return "run", world


def torchrun_command(gpus, argv, port):
    """The torchrun command line that runs this script as ``gpus`` ranks."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", str(gpus),
            "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__)] + list(argv)


def _free_port():
    import socket
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def init_dist(world, backend):
    if world <= 1:
        return None
    import datetime
    import torch.distributed as dist
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


HOLD_CYCLES = 2_000_000   # about 1 ms at the B200's 1965 MHz SM clock


def aggregate(elapsed_s, units, dist=None, device=None):
    """Whole-job throughput: sum of units over ranks / max of device time over
    ranks.  Returns (value, max_elapsed_s, total_units)."""
    if dist is None:
        return units / elapsed_s, elapsed_s, units
    t = torch.tensor([elapsed_s], dtype=torch.float64, device=device)
    u = torch.tensor([units], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(u, op=dist.ReduceOp.SUM)
    return float(u.item() / t.item()), float(t.item()), float(u.item())


# ---------------------------------------------------------------------------
# measurement helpers
# ---------------------------------------------------------------------------
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """Samples SM clocks and throttle reasons through NVML while running."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100,
    }

    def __init__(self, device_index, period_s=0.0005):
        self.period = period_s
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = None
            try:  # the NVML handle of the same physical GPU as the CUDA device
                pr = torch.cuda.get_device_properties(device_index)
                bus = "%08x:%02x:%02x.0" % (pr.pci_domain_id, pr.pci_bus_id, pr.pci_device_id)
                self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self._reasons_fn = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                getattr(pynvml, "nvmlDeviceGetCurrentClocksThrottleReasons")
        except Exception as e:  # no NVML: report that instead of clocks
            self.nv = None
            self.err = str(e)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= int(self._reasons_fn(self.h))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t is not None:
            self._t.join()

    def report(self):
        if self.nv is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable: " + self.err]}
        names = [k for k, v in self.REASONS.items() if self.reasons & v]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples)}


def source_hash(paths):
    h = hashlib.sha256()
    for p in paths:
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_record(key, src_paths):
    """DRAM bytes per launch of a kernel on one workload ("kernel:workload")
    from a committed ncu summary, only if the kernel's sources are unchanged
    since the counters were taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f).get(key)
    if not rec or rec.get("source_hash") != source_hash(src_paths):
        return None
    return rec


# ---------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------
def scan_bytes(c):
    """Algorithmic bytes of one chunked-scan call: every input once, every
    output once, plus the final states (h, prev_Bx, angle).  B and C are read
    once per group (G groups, K rotated pairs)."""
    Bt, T, H, P, N, R = c["batch"], c["seqlen"], c["nheads"], c["headdim"], c["dstate"], c["rank"]
    G, K = c.get("ngroups", 0) or H, c.get("rope_pairs", 0) or N // 2
    es = 2 if c["dtype"] == "bf16" else 4
    per_token_head = es * P + 4 + 4 + 4 * K + es * P
    per_token_group = 2 * es * R * N
    states = Bt * H * (2 * N * P * 4 + K * 4)
    params = H * 8 + (2 * H * R * P * 4 if R > 1 else 0)
    return Bt * T * (H * per_token_head + G * per_token_group) + states + params


def scan_flops(c):
    """Causal-lower-triangle flops of the chunked form (the dense work it
    skips is not counted): per chunk 2*pairs*R^2*(N+P) + 4*Q*R*N*P + 2*N*P."""
    Bt, T, H, P, N, R, Q = (c["batch"], c["seqlen"], c["nheads"], c["headdim"], c["dstate"], c["rank"],
                            c["chunk"])
    total = 0
    for t0 in range(0, T, Q):
        L = min(Q, T - t0)
        pairs = L * (L + 1) // 2
        total += 2 * pairs * R * R * (N + P) + 4 * L * R * N * P + 2 * N * P
    return Bt * H * total


def decode_bytes(c):
    """Algorithmic bytes of one decode step: the carried state read and written
    once, the per-token inputs read once, y written once (W_x, W_y once per
    head)."""
    Bt, H, P, N, R = c["batch"], c["nheads"], c["headdim"], c["dstate"], c["rank"]
    es = 2
    if c.get("state") == "factored":   # h, b_prev (R, N), x_prev (P)
        state = 2 * N * P * 4 + 2 * R * N * 4 + 2 * P * 4
    else:                              # h, prev_Bx
        state = 2 * 2 * N * P * 4
    per_lane = state + 2 * (N // 2) * 4 + es * P + 2 * es * R * N + 8 + 4 * (N // 2) + es * P
    return Bt * H * per_lane + (2 * H * R * P * 4 if R > 1 else 0)


class ScanWorkload:
    def __init__(self, idx, device):
        from state_space_lm_b200 import m3
        self.m3 = m3
        self.c = dict(gen.CONFIGS[idx])
        self.idx = idx
        c = self.c
        self.host = gen.config_inputs(idx)
        self.host.pop("generator")
        self.dev = {k: v.to(device) for k, v in self.host.items() if isinstance(v, torch.Tensor)}
        Bt, T, H, P, N = c["batch"], c["seqlen"], c["nheads"], c["headdim"], c["dstate"]
        self.G, self.K = c.get("ngroups", 0) or H, c.get("rope_pairs", 0) or N // 2
        self.out = (torch.empty(Bt, T, H, P, device=device, dtype=self.dev["x"].dtype),
                    torch.empty(Bt, H, N, P, device=device), torch.empty(Bt, H, N, P, device=device),
                    torch.empty(Bt, H, self.K, device=device))
        self.mimo = c["rank"] > 1
        d = self.m3.Dims(Bt, T, H, P, N, c["rank"], c["chunk"], self.G, self.K)
        which = self.m3.M3_WS_MIMO if self.mimo else self.m3.M3_WS_SISO
        nws = self.m3.workspace_bytes(which, d, self.m3.M3_BF16 if c["dtype"] == "bf16" else self.m3.M3_F32)
        self.ws = torch.empty(max(nws, 16), dtype=torch.uint8, device=device)
        self.units = Bt * T                       # tokens (b, t), all heads
        self.bytes = scan_bytes(c)
        self.flops = scan_flops(c)
        tc = (c["dtype"] == "bf16" and c["rank"] in (1, 2, 4) and c["headdim"] == 64 and c["dstate"] == 128
              and c["chunk"] % (64 // c["rank"]) == 0 and self.K % 4 == 0)
        self.kernel = "k_scan_tc" if tc else "k_scan_simt"
        self.srcs = [os.path.join(ROOT, "state_space_lm_b200", "csrc", self.kernel + ".cu")]
        # long sequences over few lanes run as three launches (state-only pass,
        # segment combine, full pass); the timed unit is then the whole call
        self.kernel_label = self.kernel if nws == 0 else self.kernel + " (3 passes: state, combine, full)"
        self.input_bytes = sum(v.numel() * v.element_size() for v in self.dev.values())

    def step(self, dev=None, out=None, stream=None):
        d = self.dev if dev is None else dev
        o = self.out if out is None else out
        if self.mimo:
            self.m3.mimo_chunked_fwd(d["x"], d["dt"], d["A"], d["lam"], d["theta"], d["B"], d["C"], d["D"],
                                     self.c["chunk"], W_x=d["Wx"], W_y=d["Wy"], workspace=self.ws, out=o,
                                     stream=stream)
        else:
            self.m3.siso_chunked_fwd(d["x"], d["dt"], d["A"], d["lam"], d["theta"], d["B"], d["C"], d["D"],
                                     self.c["chunk"], workspace=self.ws, out=o, stream=stream)

    def config(self):
        c = self.c
        return {"workload": c["name"], "batch": c["batch"], "seqlen": c["seqlen"], "nheads": c["nheads"],
                "headdim": c["headdim"], "dstate": c["dstate"], "rank": c["rank"], "chunk": c["chunk"],
                "ngroups": self.G, "rope_pairs": self.K,
                "inputs": "x/B/C %s, dt/lam/theta/A/D fp32, seeded synthetic" % c["dtype"],
                "l2": "inputs larger than L2 (%.0f MB vs 126 MB), no flush" % (self.input_bytes / 1e6)}

    # ---- oracle on a bounded sample of lanes (CPU baseline) ----
    def oracle_sample(self, n_lanes, threads):
        import oracle
        c = self.c
        H = c["nheads"]
        lanes = [(i // H, i % H) for i in range(min(n_lanes, c["batch"] * H))]
        bs = sorted({b for b, _ in lanes})
        hs = sorted({h for _, h in lanes})
        sl = lambda t: t[bs[0]:bs[-1] + 1, :, hs[0]:hs[-1] + 1]
        keys = ("x", "dt", "A", "lam", "theta", "B", "C", "D")
        arr = {}
        for k in keys:
            v = self.host[k]
            arr[k] = gen.to_f64(v[hs[0]:hs[-1] + 1] if k in ("A", "D") else sl(v))
        if self.G != H:   # the sampled heads' B/C rows, one per head
            hpg = H // self.G
            for k in ("B", "C"):
                v = self.host[k][bs[0]:bs[-1] + 1]
                arr[k] = gen.to_f64(torch.stack([v[:, :, h // hpg] for h in range(hs[0], hs[-1] + 1)], 2))
        nl = len(bs) * len(hs)
        t0 = time.perf_counter()
        if self.mimo:
            for k in ("Wx", "Wy"):
                arr[k] = gen.to_f64(self.host[k][hs[0]:hs[-1] + 1])
            _, used = oracle.mimo_loop(**arr, nthreads=threads, return_threads=True)
        else:
            _, used = oracle.siso_loop(**arr, nthreads=threads, return_threads=True)
        dt = time.perf_counter() - t0
        return nl, dt, used


def bwd_bytes(c):
    """Algorithmic bytes of one backward call: the forward's inputs and dy read
    once, every gradient written once (fp32), the initial-state gradients and
    the shared parameters' gradients."""
    Bt, T, H, P, N, R = c["batch"], c["seqlen"], c["nheads"], c["headdim"], c["dstate"], c["rank"]
    G, K = c.get("ngroups", 0) or H, c.get("rope_pairs", 0) or N // 2
    es = 2 if c["dtype"] == "bf16" else 4
    per_token_head = 2 * es * P + 8 + 4 * K + (4 * P + 8 + 4 * K)
    per_token_group = 2 * es * R * N + 2 * 4 * R * N
    states = Bt * H * (2 * N * P * 4 + K * 4)
    params = H * 8 * 2 + (4 * H * R * P * 4 if R > 1 else 0)
    return Bt * T * (H * per_token_head + G * per_token_group) + states + params


def bwd_flops(c):
    """Causal flops of the chunked backward at the workload's chunk Q: per chunk
    12 Q R N P (the entering-state pass and the five chunk-by-state products)
    plus 2 pairs R^2 (3N + 2P) for the masked score products (+ 2 pairs R^2 P
    for the MIMO output when W_y's gradient is wanted)."""
    Bt, T, H, P, N, R, Q = (c["batch"], c["seqlen"], c["nheads"], c["headdim"], c["dstate"], c["rank"],
                            c["chunk"])
    total = 0
    for t0 in range(0, T, Q):
        L = min(Q, T - t0)
        pairs = L * (L + 1) // 2
        total += 12 * L * R * N * P + 2 * pairs * R * R * (3 * N + 2 * P + (P if R > 1 else 0))
    return Bt * H * total


FFMA_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12   # SMs x FP32 lanes x 2 flops x max SM clock


class BwdWorkload(ScanWorkload):
    """One backward call of a chunked-scan workload: every input gradient
    from dy (the final-state adjoints zero), outputs preallocated."""

    def __init__(self, idx, device):
        super().__init__(idx, device)
        c = self.c
        self.host["dy"] = gen.grad_seed(self.host["x"], gen.SEED_BASE + 1000 + idx)
        self.dev["dy"] = self.host["dy"].to(device)
        Bt, T, H, P, N, R = c["batch"], c["seqlen"], c["nheads"], c["headdim"], c["dstate"], c["rank"]
        d = self.m3.Dims(Bt, T, H, P, N, R if self.mimo else 1, c["chunk"], self.G, self.K)
        nws = self.m3.workspace_bytes(self.m3.M3_WS_BWD_MIMO if self.mimo else self.m3.M3_WS_BWD_SISO, d,
                                      self.m3.M3_BF16 if c["dtype"] == "bf16" else self.m3.M3_F32)
        self.ws = torch.empty(max(nws, 16), dtype=torch.uint8, device=device)
        self.grads = self.m3.chunked_bwd(*[self.dev[k] for k in ("x", "dt", "A", "lam", "theta", "B", "C", "D")],
                                         self.dev["dy"], c["chunk"], W_x=self.dev.get("Wx"),
                                         W_y=self.dev.get("Wy"), workspace=self.ws)
        self.out = tuple(self.grads.values())
        self.bytes = bwd_bytes(c)
        self.flops = bwd_flops(c)
        self.kernel = "k_bwd_chunks"
        self.kernel_label = "k_bwd_state + k_bwd_chunks + k_bwd_params (3 launches)"
        self.srcs = [os.path.join(ROOT, "state_space_lm_b200", "csrc", "k_scan_bwd.cu")]
        self.input_bytes += self.host["dy"].numel() * self.host["dy"].element_size()

    def step(self, dev=None, out=None, stream=None):
        d = self.dev if dev is None else dev
        self.m3.chunked_bwd(*[d[k] for k in ("x", "dt", "A", "lam", "theta", "B", "C", "D")], d["dy"],
                            self.c["chunk"], W_x=d.get("Wx"), W_y=d.get("Wy"), out=self.grads, workspace=self.ws,
                            stream=stream)

    def config(self):
        cfg = super().config()
        cfg["pass"] = "backward: all input gradients from dy (final-state adjoints zero), fp32 gradients"
        return cfg

    def oracle_sample(self, n_lanes, threads):
        """The oracle's reverse sweep (one thread) on the first n lanes."""
        import oracle
        c = self.c
        H = c["nheads"]
        n = min(n_lanes, c["batch"] * H)
        t0 = time.perf_counter()
        for i in range(n):
            b, h = i // H, i % H
            lane = {k: gen.to_f64(self.host[k][b:b + 1, :, h:h + 1])
                    for k in ("x", "dt", "lam", "theta", "B", "C")}
            lane["A"], lane["D"] = gen.to_f64(self.host["A"][h:h + 1]), gen.to_f64(self.host["D"][h:h + 1])
            oracle.loop_bwd(**lane, dy=gen.to_f64(self.host["dy"][b:b + 1, :, h:h + 1]))
        return n, time.perf_counter() - t0, 1


def prep_bytes(c):
    """Algorithmic bytes of one standalone prep pass over a whole workload.
    Discretize: dt, lam in (8 B) and alpha, beta, gamma out (12 B) per
    token-head, A once.  Rope: B, C in and the rotated B, C out (one row per
    head), theta and dt in, per token-head; the final angle out per lane."""
    Bt, T, H, N, R = c["batch"], c["seqlen"], c["nheads"], c["dstate"], c["rank"]
    G, K = c.get("ngroups", 0) or H, c.get("rope_pairs", 0) or N // 2
    es = 2 if c["dtype"] == "bf16" else 4
    if c["prep"] == "discretize":
        return Bt * T * H * 20 + H * 4
    per_token_head = 2 * es * R * N + 4 * K + 4
    per_token_group = 2 * es * R * N
    return Bt * T * (H * per_token_head + G * per_token_group) + Bt * H * K * 4


class PrepWorkload(ScanWorkload):
    """One standalone S1 (m3_discretize) or S2 (m3_rope_bc) call over the
    default workload's inputs, outputs preallocated."""

    def __init__(self, idx, device):
        from state_space_lm_b200 import m3
        self.m3 = m3
        self.c = c = dict(gen.CONFIGS[idx])
        self.idx = idx
        self.host = gen.config_inputs(idx)
        self.host.pop("generator")
        self.dev = {k: v.to(device) for k, v in self.host.items() if isinstance(v, torch.Tensor)}
        Bt, T, H, N = c["batch"], c["seqlen"], c["nheads"], c["dstate"]
        self.G, self.K = c.get("ngroups", 0) or H, c.get("rope_pairs", 0) or N // 2
        self.mimo = False
        self.units = Bt * T
        self.kind = c["prep"]
        d = self.dev
        if self.kind == "discretize":
            self.out = tuple(torch.empty_like(d["dt"]) for _ in range(3))
            self.kernel = "k_discretize"
        else:
            self.out = (torch.empty(Bt, T, H, N, device=device, dtype=d["B"].dtype),
                        torch.empty(Bt, T, H, N, device=device, dtype=d["B"].dtype),
                        torch.empty(Bt, H, self.K, device=device))
            self.kernel = "k_rope"
        self.kernel_label = self.kernel
        self.srcs = [os.path.join(ROOT, "state_space_lm_b200", "csrc", "k_elementwise.cu")]
        self.bytes = prep_bytes(c)
        self.flops = 0
        keys = ("dt", "A", "lam") if self.kind == "discretize" else ("B", "C", "theta", "dt")
        self.host = {k: self.host[k] for k in keys}
        self.input_bytes = sum(self.host[k].numel() * self.host[k].element_size() for k in keys)

    def step(self, dev=None, out=None, stream=None):
        d = self.dev if dev is None else dev
        o = self.out if out is None else out
        if self.kind == "discretize":
            self.m3.discretize(d["dt"], d["A"], d["lam"], out=o, stream=stream)
        else:
            self.m3.rope_bc(d["B"], d["C"], d["theta"], d["dt"], out=o, stream=stream)

    def config(self):
        cfg = super().config()
        cfg.pop("chunk", None)
        cfg["pass"] = ("S1 alone: alpha, beta, gamma of every token-head" if self.kind == "discretize" else
                       "S2 alone: rotated B, C (one row per head) and the final angle")
        cfg["inputs"] = ("dt/lam/A fp32, seeded synthetic" if self.kind == "discretize" else
                         "B/C %s, theta/dt fp32, seeded synthetic" % self.c["dtype"])
        return cfg

    def oracle_sample(self, n_lanes, threads):
        """The oracle's S1 or S2 on the first batch rows holding n lanes."""
        import oracle
        c = self.c
        H = c["nheads"]
        nb = max(1, min(c["batch"], n_lanes // H))
        a = {k: gen.to_f64(v[:nb] if k != "A" else v) for k, v in self.host.items()}
        t0 = time.perf_counter()
        if self.kind == "discretize":
            oracle.discretize(a["dt"], a["A"], a["lam"])
        else:
            oracle.rope_bc(a["B"], a["C"], a["theta"], a["dt"])
        return nb * H, time.perf_counter() - t0, 1


def decode_config(c):
    """The config dict of a decode workload's bench line (both arms)."""
    factored = c.get("state") == "factored"
    state_bytes = (1 if factored else 2) * c["batch"] * c["nheads"] * c["dstate"] * c["headdim"] * 4
    return {"workload": c["name"], "batch": c["batch"], "nheads": c["nheads"], "headdim": c["headdim"],
            "dstate": c["dstate"], "prefill": c["seqlen"], "decode_steps_per_call": 1,
            "rank": c["rank"], "state": "factored (h, b_prev, x_prev)" if factored else "full (h, prev_Bx)",
            "inputs": "x/B/C bf16, dt/lam/theta fp32 per step; fp32 state and angle",
            "l2": "state larger than L2 (%.0f MB vs 126 MB), no flush" % (state_bytes / 1e6)}


class DecodeWorkload:
    """Decode steps: every step advances all (batch, head) lanes by one token.
    The carried state comes from a seeded prefill (a chunked forward over the
    first ``seqlen`` tokens, untimed; for the factored state, its last token's
    rotated B and x); the per-step inputs of every step are drawn up front and
    resident in HBM."""

    def __init__(self, idx, device, nsteps):
        from state_space_lm_b200 import m3
        self.m3 = m3
        self.c = dict(gen.CONFIGS[idx])
        c = self.c
        Bt, H, P, N = c["batch"], c["nheads"], c["headdim"], c["dstate"]
        inp = gen.config_inputs(idx)
        g = inp.pop("generator")
        self.host_prefill = inp
        d = {k: v.to(device) for k, v in inp.items() if isinstance(v, torch.Tensor)}
        R = c["rank"]
        self.factored = c.get("state") == "factored"
        self.Wx, self.Wy = d.get("Wx"), d.get("Wy")
        if R == 1:
            _, self.h, self.u, self.a = m3.siso_chunked_fwd(d["x"], d["dt"], d["A"], d["lam"], d["theta"],
                                                            d["B"], d["C"], d["D"], c["chunk"])
        else:
            _, self.h, self.u, self.a = m3.mimo_chunked_fwd(d["x"], d["dt"], d["A"], d["lam"], d["theta"],
                                                            d["B"], d["C"], d["D"], c["chunk"], W_x=self.Wx,
                                                            W_y=self.Wy)
        if self.factored:
            Br, _, _ = m3.rope_bc(d["B"], d["C"], d["theta"], d["dt"])
            last = Br[:, -1]
            self.bp = (last[:, :, None] if R == 1 else last).float().contiguous()
            self.xp = d["x"][:, -1].float().contiguous()
            self.u = None
        self.A, self.D = d["A"], d["D"]
        self.steps_host = [gen.decode_step_inputs(g, Bt, H, P, N, rank=R, rank_axis=self.factored)
                           for _ in range(nsteps)]
        self.steps_dev = [{k: v.to(device) for k, v in st.items()} for st in self.steps_host]
        self.y = torch.empty(Bt, H, P, device=device, dtype=torch.bfloat16)
        self.i = 0
        self.units = Bt                           # one token per sequence per step
        self.bytes = decode_bytes(c)
        self.flops = 0
        self.kernel = self.kernel_label = "k_decode_gen" if (self.factored or R > 1) else "k_decode"
        self.srcs = [os.path.join(ROOT, "state_space_lm_b200", "csrc", "k_decode.cu")]
        self.input_bytes = (1 if self.factored else 2) * Bt * H * N * P * 4

    def step(self, dev=None, out=None, stream=None):
        st = self.steps_dev[self.i % len(self.steps_dev)] if dev is None else dev
        self.i += 1
        y = self.y if out is None else out
        if self.factored:
            self.m3.step_decode_factored(st["x"], st["dt"], self.A, st["lam"], st["theta"], st["B"], st["C"],
                                         self.D, self.h, self.bp, self.xp, self.a, W_x=self.Wx, W_y=self.Wy,
                                         y_out=y, stream=stream)
        elif self.c["rank"] > 1:
            self.m3.mimo_step_decode(st["x"], st["dt"], self.A, st["lam"], st["theta"], st["B"], st["C"], self.D,
                                     self.h, self.u, self.a, W_x=self.Wx, W_y=self.Wy, y_out=y, stream=stream)
        else:
            self.m3.step_decode(st["x"], st["dt"], self.A, st["lam"], st["theta"], st["B"], st["C"], self.D,
                                self.h, self.u, self.a, y_out=y, stream=stream)

    def config(self):
        return decode_config(self.c)


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def run_cpu_baseline(w, target_s=10.0, wall_s=1.5):
    """Time the oracle as it stands on the host cores on a bounded sample of
    lanes; tokens/s are scaled to whole (b, t) tokens of all heads."""
    cores = os.cpu_count() or 1
    H = w.c["nheads"]
    total_lanes = w.c["batch"] * H
    n = min(total_lanes, max(1, cores))
    nl, dt, used = w.oracle_sample(n, cores)
    if dt < target_s / 4 and nl < total_lanes:
        n = int(min(total_lanes, nl * max(1.0, target_s / max(dt, 1e-3))))
        n = max(H, (n // H) * H)
        nl, dt, used = w.oracle_sample(n, cores)
    reps = 1
    if nl == total_lanes and dt < wall_s:
        # the whole workload is quick: repeat it for a steadier figure
        reps = int(min(50, max(2, round(wall_s / max(dt, 1e-3)))))
        dt, used2 = 0.0, used
        for _ in range(reps):
            _, d1, used2 = w.oracle_sample(n, cores)
            dt += d1
        used = used2
    tokens = reps * nl * w.c["seqlen"] / H
    # one thread on one lane (a prep pass: one batch row), scaled to whole
    # tokens of all heads
    nl1, d1, _ = w.oracle_sample(1, 1)
    return {"value": tokens / dt, "unit": UNIT, "cores": int(used), "kind": "oracle",
            "sample": "%d x %d of %d (b,h) lanes x %d tokens, fp64 C loop, %.1f s wall on %d threads"
                      % (reps, nl, total_lanes, w.c["seqlen"], dt, used),
            "one_thread_value": nl1 * w.c["seqlen"] / H / d1, "cpu_model": cpu_model()}


def decode_oracle_sample(c, nb, steps, threads):
    """The oracle's decode step (the one the workload's kernel computes: full
    state, rank R, or factored) over `steps` steps of the first nb sequences,
    all heads, from a zero state (the time does not depend on the values).
    Returns (sequences x steps, seconds, threads used)."""
    import oracle
    H, P, N, R = c["nheads"], c["headdim"], c["dstate"], c["rank"]
    factored = c.get("state") == "factored"
    # the parameters and per-step inputs of the workload's shape, drawn small
    # (the full prefill is not needed: the time does not depend on the values)
    inp = gen.scan_inputs(1, 1, H, P, N, rank=R, dtype=c["dtype"], seed=gen.SEED_BASE + 77,
                          mimo_weights=R > 1)
    g = inp.pop("generator")
    A, D = gen.to_f64(inp["A"]), gen.to_f64(inp["D"])
    Wx = gen.to_f64(inp["Wx"]) if R > 1 else None
    Wy = gen.to_f64(inp["Wy"]) if R > 1 else None
    st = [gen.decode_step_inputs(g, nb, H, P, N, rank=R, rank_axis=factored) for _ in range(steps)]
    st = [{k: gen.to_f64(v) for k, v in s.items()} for s in st]
    h, u = np.zeros((nb, H, N, P)), np.zeros((nb, H, N, P))
    a = np.zeros((nb, H, N // 2))
    bp, xp = np.zeros((nb, H, R, N)), np.zeros((nb, H, P))
    t0 = time.perf_counter()
    for s in st:
        args = (s["x"], s["dt"], A, s["lam"], s["theta"], s["B"], s["C"], D)
        if factored:
            _, h, bp, xp, a = oracle.step_decode_factored(*args, h, bp, xp, a, Wx=Wx, Wy=Wy)
        elif R > 1:
            _, h, u, a = oracle.mimo_step_decode(*args, h, u, a, Wx=Wx, Wy=Wy, nthreads=threads)
        else:
            _, h, u, a = oracle.step_decode(*args, h, u, a, nthreads=threads)
    used = 1 if factored else min(threads, nb * H)
    return nb * steps, time.perf_counter() - t0, used


def run_cpu_baseline_decode(c, target_s=6.0):
    cores = os.cpu_count() or 1
    nb = min(c["batch"], 16)
    n, dt, used = decode_oracle_sample(c, nb, 2, cores)
    steps = int(max(2, min(200, 2 * target_s / max(dt, 1e-3))))
    n, dt, used = decode_oracle_sample(c, nb, steps, cores)
    return {"value": n / dt, "unit": UNIT, "cores": int(used), "kind": "oracle",
            "sample": "%d decode steps of %d of %d sequences (all heads), fp64 C step, %.1f s on %d threads"
                      % (steps, nb, c["batch"], dt, used)}


def run_cpu_baseline_bwd(w, target_s=8.0):
    """The oracle's backward (single-threaded C loop) on as many lanes as fit
    about target_s seconds; tokens/s scaled to whole (b, t) tokens."""
    H = w.c["nheads"]
    nl, dt, _ = w.oracle_sample(1, 1)
    n = int(min(w.c["batch"] * H, max(1, target_s / max(dt, 1e-3))))
    if n > 1:
        nl, dt, _ = w.oracle_sample(n, 1)
    tokens = nl * w.c["seqlen"] / H
    return {"value": tokens / dt, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": "%d of %d (b,h) lanes x %d tokens, fp64 reverse sweep, %.1f s on 1 thread"
                      % (nl, w.c["batch"] * H, w.c["seqlen"], dt)}


# ---------------------------------------------------------------------------
# the two arms
# ---------------------------------------------------------------------------
def run_ours(args, world, rank, local):
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    dist = init_dist(world, "nccl")
    from state_space_lm_b200 import build, m3
    if not os.path.exists(build.LIB):
        raise SystemExit("CUDA library not built: run python -m state_space_lm_b200.build")
    if "steps" in gen.CONFIGS[args.config]:      # the decode workloads
        w = DecodeWorkload(args.config, device, args.steps + args.warmup)
    elif gen.CONFIGS[args.config].get("grad"):
        w = BwdWorkload(args.config, device)
    elif gen.CONFIGS[args.config].get("prep"):
        w = PrepWorkload(args.config, device)
    else:
        w = ScanWorkload(args.config, device)
    stream = torch.cuda.current_stream(device)

    for _ in range(args.warmup):
        w.step()
    torch.cuda.synchronize(device)

    # ---- device-timed region: K steps back to back, inputs resident in HBM ----
    # One event before the first step and one after the last, on the launching
    # stream: a pair of events around every step would put two event writes
    # between consecutive launches (about 5 % of a 0.1 ms step, measured).  The
    # average launch time of a one-launch step is then the region time / K; a
    # step of several launches reports the whole call.
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(device)
    n0 = m3.launch_count()
    start = torch.cuda.Event(enable_timing=True)
    stop = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        # hold the stream for about a millisecond (a bounded spin kernel), so
        # that the first steps are queued while it runs: the events then time
        # the K steps on the device, not the host's first launch (the binding's
        # checks, the tensor-map encoding) or the sampler thread's start-up;
        # the e2e number below counts the host side
        with torch.cuda.stream(stream):
            torch.cuda._sleep(HOLD_CYCLES)
        start.record(stream)
        for i in range(args.steps):
            w.step()
        stop.record(stream)
        torch.cuda.synchronize(device)
    launches = m3.launch_count() - n0
    if dist is not None:
        dist.barrier()
    elapsed = start.elapsed_time(stop) / 1e3
    kernel_s = elapsed / args.steps
    value, tmax, units = aggregate(elapsed, w.units * args.steps, dist, device)

    # ---- end to end through the C ABI with host buffers ----
    e2e_steps = max(3, min(args.steps, 20))
    if isinstance(w, DecodeWorkload):
        pinned = [{k: v.pin_memory() for k, v in st.items()} for st in w.steps_host[:e2e_steps]]
        stage = {k: torch.empty_like(v) for k, v in w.steps_dev[0].items()}
        hy = torch.empty(w.y.shape, dtype=w.y.dtype).pin_memory()
        h2d = sum(v.numel() * v.element_size() for v in pinned[0].values())
        d2h = hy.numel() * hy.element_size()
        e2e_i = [0]

        def e2e_step():
            src = pinned[e2e_i[0] % len(pinned)]
            e2e_i[0] += 1
            for k, v in src.items():
                stage[k].copy_(v, non_blocking=True)
            w.step(dev=stage)
            hy.copy_(w.y, non_blocking=True)
    else:
        pinned = {k: v.pin_memory() for k, v in w.host.items() if isinstance(v, torch.Tensor)}
        hout = tuple(torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in w.out)
        h2d = sum(v.numel() * v.element_size() for v in pinned.values())
        d2h = sum(o.numel() * o.element_size() for o in hout)

        def e2e_step():
            for k, v in pinned.items():
                w.dev[k].copy_(v, non_blocking=True)
            w.step()
            for o, ho in zip(w.out, hout):
                ho.copy_(o, non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize(device)
    if dist is not None:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(device)
    e2e_val, _, _ = aggregate(e0.elapsed_time(e1) / 1e3, w.units * e2e_steps, dist, device)

    peaks, peak_kind = load_peaks()
    achieved = w.bytes / kernel_s / 1e9
    tr = traffic_record(w.kernel + ":" + w.c["name"], w.srcs)
    if isinstance(w, BwdWorkload):
        # FFMA-bound: flops against the FP32 pipes' peak (148 SMs x 128 lanes x 2 x 1.965 GHz)
        ach = w.flops / kernel_s / 1e12
        roof = {"bound": "alu", "achieved": round(ach, 2), "peak": round(FFMA_PEAK_TFLOPS, 1), "unit": "TFLOP/s",
                "frac": round(ach / FFMA_PEAK_TFLOPS, 4), "traffic": (tr["dram_bytes_per_launch"] if tr else None),
                "kernel": w.kernel_label, "algorithmic_flops": w.flops, "algorithmic_bytes": w.bytes,
                "hbm_gbs": round(achieved, 1), "kernel_ms": round(kernel_s * 1e3, 4),
                "peak_source": "derived: 148 SMs x 128 FP32 lanes x 2 flops x 1965 MHz (no measured FP32 peak)"}
    else:
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / peaks["hbm_gbs"], 4),
                "traffic": (tr["dram_bytes_per_launch"] if tr else None),
                "kernel": w.kernel_label, "algorithmic_bytes": w.bytes,
                "kernel_ms": round(kernel_s * 1e3, 4),
                "tensor_tflops": round(w.flops / kernel_s / 1e12, 2),
                "peak_source": "%s (MEASURED_PEAKS.json hbm_gbs)" % peak_kind if peak_kind == "measured"
                else "fallback 6.65 TB/s"}

    line = {"metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(tmax / args.steps * 1e3, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.c["dtype"],
            "data": "synthetic (seeded; shapes of the pages' 434M-class layers)",
            "config": dict(w.config(), parallelism="replicas x%d (independent lanes, no collective)" % world),
            "roofline": roof,
            "e2e": {"value": round(e2e_val, 1), "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "clocks": clk.report(), "gpu_launches": int(launches)}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        if isinstance(w, DecodeWorkload):
            line["cpu_baseline"] = run_cpu_baseline_decode(w.c)
        else:
            line["cpu_baseline"] = (run_cpu_baseline_bwd(w) if isinstance(w, BwdWorkload) else run_cpu_baseline(w))
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def run_reference(args, world, rank):
    """The oracle arm: fp64 CPU loop on the host cores, a bounded sample of the
    workload per step.  Under torchrun only rank 0 runs it."""
    if rank != 0:
        return
    import oracle
    oracle.build_oracle()
    if "steps" in gen.CONFIGS[args.config]:      # decode workloads: the oracle's decode step
        run_reference_decode(args, world)
        return
    bwd = bool(gen.CONFIGS[args.config].get("grad"))
    prep = gen.CONFIGS[args.config].get("prep")
    cls = BwdWorkload if bwd else (PrepWorkload if prep else ScanWorkload)
    w = cls.__new__(cls)
    w.c = dict(gen.CONFIGS[args.config])
    w.idx = args.config
    w.host = gen.config_inputs(args.config)
    w.host.pop("generator")
    if prep:
        w.kind = prep
    if bwd:
        w.host["dy"] = gen.grad_seed(w.host["x"], gen.SEED_BASE + 1000 + args.config)
    w.mimo = w.c["rank"] > 1
    w.G = w.c.get("ngroups", 0) or w.c["nheads"]
    w.K = w.c.get("rope_pairs", 0) or w.c["dstate"] // 2
    # the same config dict as the GPU arm's line (input bytes from the host copies)
    keys = (("dt", "A", "lam") if prep == "discretize" else ("B", "C", "theta", "dt")) if prep else \
        [k for k, v in w.host.items() if isinstance(v, torch.Tensor)]
    w.input_bytes = sum(w.host[k].numel() * w.host[k].element_size() for k in keys)
    cores = os.cpu_count() or 1
    H = w.c["nheads"]
    total_lanes = w.c["batch"] * H
    n = min(total_lanes, max(H, (cores // H) * H if cores >= H else H))
    if bwd:
        n = 2    # the reverse sweep is single-threaded: two lanes per step
    for _ in range(args.warmup):
        w.oracle_sample(n, cores)
    times = []
    used = cores
    for _ in range(args.steps):
        nl, dt, used = w.oracle_sample(n, cores)
        times.append(dt)
    tokens = nl * w.c["seqlen"] / H
    el = sum(times)
    value = tokens * args.steps / el
    sample = "%d of %d (b,h) lanes x %d tokens per step, fp64 C %s" % (
        nl, total_lanes, w.c["seqlen"], "reverse sweep, 1 thread" if bwd else "loop")
    c = w.c
    line = {"metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(el / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": dict(w.config(), parallelism="replicas x%d (independent lanes, no collective)" % world),
            "impl": "reference",
            "cpu_baseline": {"value": round(value, 1), "unit": UNIT, "cores": int(used), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 1), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_reference_decode(args, world):
    c = dict(gen.CONFIGS[args.config])
    cores = os.cpu_count() or 1
    nb = min(c["batch"], 16)
    for _ in range(args.warmup):
        decode_oracle_sample(c, nb, 1, cores)
    n, el, used = decode_oracle_sample(c, nb, args.steps, cores)
    value = n / el
    line = {"metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(el / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": dict(decode_config(c), parallelism="replicas x%d (independent lanes, no collective)" % world),
            "impl": "reference",
            "cpu_baseline": {"value": round(value, 1), "unit": UNIT, "cores": int(used), "kind": "oracle",
                             "sample": "%d of %d sequences (all heads) per decode step, fp64 C step"
                                       % (nb, c["batch"])},
            "e2e": {"value": round(value, 1), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", type=int, default=1, choices=sorted(gen.CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    plan, what = launch_plan(args.gpus, os.environ)
    if plan == "error":
        raise SystemExit("bench.py: " + what)
    if plan == "relaunch":
        import subprocess
        raise SystemExit(subprocess.call(torchrun_command(what, sys.argv[1:], _free_port())))
    world, rank, local = dist_env()
    if args.impl == "reference":
        run_reference(args, world, rank)
    else:
        run_ours(args, world, rank, local)


if __name__ == "__main__":
    main()
