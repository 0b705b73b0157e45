"""Benchmark of the SAS hot path on B200.

One step = one pass of the whole training-side path over one batch of the
Qwen3-8B-like layer (B=2, Hq=32, Hkv=8, d=128, T=32768, block 64, K=32 blocks,
Student-t selector scores): gate normalisation fused with Top-K threshold
selection, forward, backward (dQ/dK/dV/dLogG) and the selector-score gradient
ds. The metric is attended-block TFLOP/s: 4*d*sum_rows(n_t) for the forward and
2.5x that for the backward, n_t = (t mod 64) + 1 + 64*min(K-1, c_t) attended keys
of row t. The same step on the Qwen3-4B-like layer (T=8192, K=16) and the
Qwen3-14B-like layer (T=65536, K=16) is reported in "legs", and the
memory-bound decode step (16 sequences over a 32768-token cache) in GB/s.

Usage:
  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
Multi-GPU: launched by torchrun, one process per GPU; each rank runs a replica
of the step on its own batch (inputs seeded by the rank; no collective on the
data path: the work splits into independent (batch, KV-group) units), and the
timed region is reduced with max over ranks.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from gated_block_sparse_flashattention_b200 import workloads  # noqa: E402

# DRAM bytes per call (dram__bytes_read.sum + dram__bytes_write.sum of the call's kernels, from one ncu
# capture, cold caches), reported as the roofline "traffic" only while the kernel sources still match the
# ones measured (sha256 prefixes); after any change they read as unmeasured (null). Keys: call:workload. The
# paged decode was captured on its 64K-token pool only (the 512K pool is too large to capture), so the 512K
# leg reports no traffic.
_BWD_SRC = {"sas_bwd_gather.cu": "d66885ea749f6bbe", "sas_lists.cu": "c8917b447428d9c8",
            "sas_common.cuh": "ff1aecbd563f87e0"}
_DEC_SRC = {"sas_decode.cu": "fa84e521f2e8049d", "sas_common.cuh": "ff1aecbd563f87e0"}
# The paged capture was taken on an earlier revision of the decode source (its three-kernel path unchanged since).
_PAGED_SRC = {"sas_decode.cu": "cef46c6cf5d95522", "sas_common.cuh": "ff1aecbd563f87e0"}
MEASURED_TRAFFIC = {
    "sas_bwd:qwen3_8b_t32k": (19891369216, _BWD_SRC),
    "sas_bwd:qwen3_4b_t8k": (2421301824, _BWD_SRC),
    "decode:decode_b16_l32k": (67838080, _DEC_SRC),
    "decode_paged:decode_b8_l64k_paged": (72023680, _PAGED_SRC),
}


def measured_traffic(name: str):
    import hashlib

    nbytes, sources = MEASURED_TRAFFIC[name]
    csrc = os.path.join(ROOT, "gated_block_sparse_flashattention_b200", "csrc")
    for fname, digest in sources.items():
        with open(os.path.join(csrc, fname), "rb") as f:
            if hashlib.sha256(f.read()).hexdigest()[:16] != digest:
                return None
    return nbytes


BENCH_WORKLOAD = "qwen3_8b_t32k"
LEG_WORKLOADS = ("qwen3_4b_t8k", "qwen3_14b_t64k")
VARLEN_WORKLOAD = "qwen3_4b_t8k"
DECODE_WORKLOAD = "decode_b16_l32k"
PAGED_DECODE_WORKLOAD = "decode_b8_l512k_paged"
VARLEN_DOCS = [512, 1536, 1024, 2048, 3072]   # documents packed into the Qwen3-4B-like layer's 8192 positions
METRIC = "fwd+bwd attended-block TFLOP/s (normalise+select+fwd+bwd+gate-grad step)"
L2_FLUSH_BYTES = 512 << 20   # > 126 MB L2, written between timed steps


# ----------------------------------------------------------------------------- work counts
def attended_keys_per_row(T: int, K: int, block: int = 64) -> np.ndarray:
    """n_t for every position t: causal part of the current block plus min(K-1, c_t) full blocks."""
    t = np.arange(T)
    return (t % block) + 1 + block * np.minimum(K - 1, t // block)


def attended_flops_varlen(w, docs) -> tuple[float, float]:
    """(forward, backward) algorithmic FLOPs of one packed step: every document a sequence of its own."""
    n = sum(attended_keys_per_row(L, w.K, w.block).sum(dtype=np.float64) for L in docs)
    fwd = 4.0 * w.d * n * w.B * w.Hq
    return fwd, 2.5 * fwd


def attended_flops(w) -> tuple[float, float]:
    """(forward, backward) algorithmic FLOPs of one step of workload w."""
    n = attended_keys_per_row(w.T, w.K, w.block).sum(dtype=np.float64)
    fwd = 4.0 * w.d * n * w.B * w.Hq
    return fwd, 2.5 * fwd


SLOT_BUDGET = 8 << 30   # bytes of forward partials per batch of (b, g) groups


MERGE_LSE_CAP = 1024    # slots x heads of one row that the partials' merge takes


def fwd_uses_gather(w) -> bool:
    """Whether sas_fwd runs the KV-block-outer forward (per-pair partials of one (b, g) within the slot budget:
    T * min(K, NB+1) slots of G x (128 bf16 + one fp32), and at most MERGE_LSE_CAP slots x heads per row) or
    the q-tile union forward."""
    slots = 1 + max(0, min(w.K - 1, w.NB))
    return w.T * slots * w.G * (128 * 2 + 4) <= SLOT_BUDGET and slots * w.G <= MERGE_LSE_CAP


def executed_flops(w, sel):
    """(forward, backward) FLOPs the tensor cores execute for one step, from the selection sel [B,Hkv,T,K-1].

    KV-block-outer kernels (the backward, and the forward when its partials fit the slot budget): the CTA of
    block j runs its MMAs per tile of P positions x G heads (up to 128 rows) over the positions that attend j
    (its own 64 and those that selected it): 2 MMAs of 128 x 64 x 128 MACs per tile for the forward (S and P V),
    5 for the backward. The q-tile union forward: every q-tile (P positions x G heads) runs S = Q K^T and
    O += P V over its block list, the current block(s) plus the union of its rows' selected blocks. The ratio
    to the attended FLOPs is the waste of the tiling.
    """
    G = w.G
    P = (128 // G) & ~7
    B, Hkv, T, H = sel.shape
    nbg = B * Hkv
    mma = 2.0 * 128 * 64 * 128
    n_pt = (T + P - 1) // P
    s2 = sel.reshape(nbg, T, H).long()
    if n_pt * P > T:
        s2 = torch.cat([s2, torch.full((nbg, n_pt * P - T, H), -1, dtype=s2.dtype, device=s2.device)], 1)
    s2 = s2.reshape(nbg, n_pt, P * H) + 1                     # 0: no block
    hit = torch.zeros(nbg, n_pt, w.NB + 1, dtype=torch.bool, device=sel.device)
    hit.scatter_(2, s2, True)
    t0 = torch.arange(n_pt, device=sel.device) * P
    t1 = torch.clamp(t0 + P, max=T) - 1
    n_cur = (t1 // w.block - t0 // w.block + 1).to(torch.float64)
    fwd_union = float((hit[:, :, 1:].sum(-1).to(torch.float64) + n_cur).sum()) * 2 * mma
    del hit
    counts = torch.zeros(nbg, w.NB + 1, dtype=torch.float64, device=sel.device)
    counts.scatter_add_(1, sel.reshape(nbg, T * H).long() + 1, torch.ones(nbg, T * H, dtype=torch.float64,
                                                                        device=sel.device))
    own = torch.clamp(T - torch.arange(w.NB, device=sel.device) * w.block, max=w.block).to(torch.float64)
    tiles = float(torch.ceil((counts[:, 1:] + own) / P).sum())
    fwd = tiles * 2 * mma if fwd_uses_gather(w) else fwd_union
    bwd = tiles * 5 * mma
    return fwd, bwd


def gate_select_bytes(w, compact: bool = False, with_sel: bool = False) -> float:
    """HBM bytes of the fused normalise + select: the causal part of s read once, tau and tau_idx written, and
    the full logG row written (compact gates: the row's score LSE, 4 bytes, instead), plus the K-1 selected
    block indices of each row when the index list is written."""
    c = np.minimum(np.arange(w.T) // w.block, w.NB).astype(np.float64)
    rows = w.B * w.Hkv
    out = 4.0 * w.T if compact else 4.0 * w.NB * w.T
    sel = 4.0 * max(w.K - 1, 0) * w.T if with_sel else 0.0
    return rows * (4.0 * c.sum() + out + 8.0 * w.T + sel)


def gate_grad_bytes(w) -> float:
    """HBM bytes of the selector-score gradient: the causal parts of logG and dLogG read, the full ds row
    written."""
    c = np.minimum(np.arange(w.T) // w.block, w.NB).astype(np.float64)
    rows = w.B * w.Hkv
    return rows * (4.0 * c.sum() * 2 + 4.0 * w.NB * w.T)


def noisy_select_bytes(w) -> float:
    """HBM bytes of the noisy (full*) selection: the causal parts of logG and of the noise read, the full
    logG_sel row written, tau and tau_idx written."""
    c = np.minimum(np.arange(w.T) // w.block, w.NB).astype(np.float64)
    rows = w.B * w.Hkv
    return rows * (4.0 * c.sum() * 2 + 4.0 * w.NB * w.T + 8.0 * w.T)


def time_noisy_select(w, logG, flush, stream, binding, device, reps=10):
    """Mean device time (ms) of sas_select_noisy on the step's gates with seeded N(0, 1) noise, L2 flushed
    before each call (outside the events). Not part of the step: the full* scope replaces the plain
    selection with it."""
    gen = torch.Generator(device=device).manual_seed(7)
    noise = torch.randn(logG.shape, generator=gen, device=device)
    lsel = torch.empty_like(logG)
    tau = torch.empty(logG.shape[:3], device=device)
    tidx = torch.empty(logG.shape[:3], dtype=torch.int32, device=device)
    times = []
    for i in range(reps + 3):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        binding.sas_select_noisy(logG, noise, lsel, tau, tidx, None, w.K, stream=stream)
        b.record(stream)
        times.append((a, b))
    torch.cuda.synchronize(device)
    return statistics.mean(a.elapsed_time(b) for a, b in times[3:])


def decode_bytes(w) -> float:
    """Algorithmic bytes of one decode step: selected K/V blocks, q, o and the score rows."""
    el = 2 if w.dtype == "bf16" else 4
    kv = 2.0 * w.B * w.Hkv * w.K * w.block * w.d * el
    qo = 2.0 * w.B * w.Hq * w.d * el
    s = w.B * w.Hkv * w.NB * 4.0
    return kv + qo + s


# ----------------------------------------------------------------------------- multi-rank helpers
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def rank_inputs(w, rank: int):
    """The batch one rank works on: the workload's seeded inputs with the rank as the seed (every rank a
    replica of the step on its own data)."""
    return workloads.make_training_inputs(w, seed=rank)


def job_throughput(flops_per_step: float, steps: int, max_total_ms: float, world: int) -> float:
    """Whole-job TFLOP/s: every rank's steps, over the slowest rank's timed region."""
    return world * flops_per_step * steps / (max_total_ms * 1e-3) / 1e12


def reduce_max(value: float, device=None) -> float:
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized():
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clocks / throttle reasons, sampled every 50 ms while `active` is set (from the first
    warm-up step to the end of the decode leg). The summary keeps the samples drawn under load (power
    draw at least half of the largest seen): the timed regions themselves are tens of milliseconds."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines: list[str] = []
        self._thr = None
        self.active = False

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._thr = threading.Thread(target=self._read, daemon=True)
            self._thr.start()
        except (FileNotFoundError, OSError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            if self.active:
                self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            if self._thr:
                self._thr.join(timeout=2)

    def summary(self):
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        rows = []
        for line in self.lines:
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                rows.append((float(f[1]), float(f[2]), float(f[3]), f[5:9]))
            except ValueError:
                continue
        pmax = max((r[2] for r in rows), default=0.0)
        for clock, cmax, power, flags in rows:
            if power < 0.5 * pmax:
                continue
            sm.append(clock)
            smax = cmax
            for name, val in zip(names, flags):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ----------------------------------------------------------------------------- CPU baseline (oracle)
def oracle_sample(w, seconds: float, seed: int = 0):
    """Time the CPU oracle, as it stands, on consecutive 128-row chunks of one
    (b, g) group of workload w (the last positions: the longest rows) until
    about ``seconds`` of work. Returns (TFLOP/s, threads, description)."""
    from oracle import sas_oracle as orc

    try:
        from threadpoolctl import threadpool_info
        threads = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:  # noqa: BLE001
        threads = 1
    inp = workloads.make_training_inputs(w, seed=seed)
    f64 = lambda t: t[:1, : w.G].float().numpy().astype(np.float64)  # noqa: E731
    Q, dO = f64(inp["Q"]), f64(inp["dO"])
    Kt = inp["K"][:1, :1].float().numpy().astype(np.float64)
    V = inp["V"][:1, :1].float().numpy().astype(np.float64)
    s = inp["s"][:1, :1].numpy().astype(np.float64)
    logG = orc.gate_normalize(s, w.block)
    tau, tidx, _ = orc.select_threshold(logG, w.K, w.block)
    n_t = attended_keys_per_row(w.T, w.K, w.block)
    work, elapsed, rows_done = 0.0, 0.0, 0
    hi = w.T
    while elapsed < seconds and hi > 0:
        rows = np.arange(max(0, hi - 128), hi)
        t0 = time.perf_counter()
        orc.forward_backward(Q, Kt, V, dO, logG, tau, tidx, w.block, w.sm_scale, rows=rows)
        elapsed += time.perf_counter() - t0
        work += 3.5 * 4.0 * w.d * n_t[rows].sum() * w.G
        rows_done += len(rows)
        hi -= 128
    desc = (f"oracle fwd+bwd (materialised, fp64) on {rows_done} query positions x {w.G} heads of one "
            f"(batch, KV group) of {w.name}; gates normalised/selected by the oracle outside the timing, "
            f"selector-score gradient not sampled (O(NB) per row against O(n_t d) attention work)")
    return work / elapsed / 1e12, threads, desc


# ----------------------------------------------------------------------------- GPU arm
def workload_desc(w) -> str:
    dist = {"normal": "s~N(0,1)", "normal2_planted3": "s~N(0,2) + 3 planted blocks per query",
            "student_t3": "s~Student-t(nu=3)"}[w.s_dist]
    return (f"{w.name} layer fwd+bwd: B={w.B} Hq={w.Hq} Hkv={w.Hkv} d={w.d} T={w.T} block={w.block} K={w.K} "
            f"({w.K * w.block}-token budget), {dist}")


def run_training(w, args, device, stream, binding, peaks, rank, world, host=None, noisy=False):
    """Times the training step (fused normalise+select, fwd, bwd, selector gradient) of workload w with inputs
    resident in HBM, a 512 MiB L2 flush between steps outside the events. Returns (result dict, host inputs)."""
    fwd_flops, bwd_flops = attended_flops(w)
    step_flops = fwd_flops + bwd_flops
    if host is None:
        host = rank_inputs(w, rank)
    Q, K, V, dO, s = (host[k].to(device) for k in ("Q", "K", "V", "dO", "s"))
    # Compact gates: the fused selection keeps each row's score LSE instead of writing logG; the attention
    # and gradient calls rebuild log g = s - LSE (bit-identical to logG). The selection also writes each
    # row's sorted block list, from which the attention calls build their per-block row lists.
    gate_lse = torch.empty(w.B, w.Hkv, w.T, device=device)
    tau = torch.empty(w.B, w.Hkv, w.T, device=device)
    tidx = torch.empty(w.B, w.Hkv, w.T, dtype=torch.int32, device=device)
    sel = torch.empty(w.B, w.Hkv, w.T, max(w.K - 1, 1), dtype=torch.int32, device=device)
    O = torch.empty_like(Q)
    LSE = torch.empty(w.B, w.Hq, w.T, device=device)
    dQ, dK, dV, dLogG = torch.empty_like(Q), torch.empty_like(K), torch.empty_like(V), torch.empty_like(s)
    ds = torch.empty_like(s)
    ws_f = binding.workspace(binding.sas_fwd_workspace_size(w.B, w.Hq, w.Hkv, w.T, w.d, w.K, 1), device)
    ws_b = binding.workspace(binding.sas_bwd_workspace_size(w.B, w.Hq, w.Hkv, w.T, w.d, w.K, 1), device)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        binding.sas_gate_normalize_select_compact(s, gate_lse, tau, tidx, sel, w.K, stream=stream)
        if ev:
            ev[1].record(stream)
        binding.sas_fwd(Q, K, V, s, tau, tidx, O, LSE, w.K, w.sm_scale, ws_f, stream=stream, gate_lse=gate_lse,
                        sel=sel)
        if ev:
            ev[2].record(stream)
        binding.sas_bwd(Q, K, V, O, dO, s, tau, tidx, LSE, dQ, dK, dV, dLogG, w.K, w.sm_scale, ws_b,
                        stream=stream, gate_lse=gate_lse, sel=sel)
        if ev:
            ev[3].record(stream)
        binding.sas_gate_grad(s, dLogG, ds, stream=stream, gate_lse=gate_lse)
        if ev:
            ev[4].record(stream)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize(device)
    if binding.sas_device_status(ws_f) or binding.sas_device_status(ws_b):
        raise RuntimeError(f"kernel-side error during warm-up of {w.name}")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    barrier(device)
    torch.cuda.synchronize(device)
    launches0 = binding.launch_count()
    for i in range(args.steps):
        flush.zero_()      # L2 flush between timed steps (outside the events)
        step(evs[i])
    torch.cuda.synchronize(device)
    launches = binding.launch_count() - launches0
    barrier(device)
    step_ms = [e[0].elapsed_time(e[4]) for e in evs]
    fwd_ms = [e[1].elapsed_time(e[2]) for e in evs]
    bwd_ms = [e[2].elapsed_time(e[3]) for e in evs]
    gate_ms = [e[0].elapsed_time(e[1]) for e in evs]
    grad_ms = [e[3].elapsed_time(e[4]) for e in evs]
    total_ms = reduce_max(sum(step_ms), device)
    status = binding.sas_device_status(ws_f) or binding.sas_device_status(ws_b)

    # Dominant call against the tensor-core roofline.
    bwd_avg = statistics.mean(bwd_ms)
    fwd_avg = statistics.mean(fwd_ms)
    dom_name, dom_ms, dom_flops = ("sas_bwd", bwd_avg, bwd_flops) if bwd_avg >= fwd_avg else \
        ("sas_fwd", fwd_avg, fwd_flops)
    achieved = dom_flops / (dom_ms * 1e-3) / 1e12
    torch.cuda.synchronize(device)
    ex_fwd, ex_bwd = executed_flops(w, sel)
    gate_avg = statistics.mean(gate_ms)
    grad_avg = statistics.mean(grad_ms)
    traffic_key = f"{dom_name}:{w.name}"
    roofline = {"bound": "tensor", "kernel": f"{dom_name} call", "achieved": round(achieved, 2),
                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": round(achieved / peaks["bf16_tflops"], 4),
                "traffic": measured_traffic(traffic_key) if traffic_key in MEASURED_TRAFFIC else None,
                "peak_source": f"{peaks['source']} bf16 burst (cuBLAS)",
                "fwd_path": "kv-block outer, per-pair partials + merge" if fwd_uses_gather(w) else "q-tile union",
                "fwd_ms": round(fwd_avg, 4), "bwd_ms": round(bwd_avg, 4),
                "fwd_tflops": round(fwd_flops / (fwd_avg * 1e-3) / 1e12, 2),
                "fwd_executed_tflops": round(ex_fwd / (fwd_avg * 1e-3) / 1e12, 2),
                "fwd_inflation": round(ex_fwd / fwd_flops, 3),
                "bwd_tflops": round(bwd_flops / (bwd_avg * 1e-3) / 1e12, 2),
                "bwd_executed_tflops": round(ex_bwd / (bwd_avg * 1e-3) / 1e12, 2),
                "bwd_inflation": round(ex_bwd / bwd_flops, 3),
                "gate_select": "compact (row score LSE instead of logG) + sorted block list per row",
                "gate_select_ms": round(gate_avg, 4),
                "gate_select_bytes": gate_select_bytes(w, compact=True, with_sel=True),
                "gate_select_bytes_with_logg": gate_select_bytes(w),
                "gate_select_gbs": round(gate_select_bytes(w, compact=True, with_sel=True) / (gate_avg * 1e-3) / 1e9,
                                         1),
                "gate_grad_ms": round(grad_avg, 4),
                "gate_grad_gbs": round(gate_grad_bytes(w) / (grad_avg * 1e-3) / 1e9, 1)}
    if noisy:
        logG = torch.empty_like(s)   # the noisy selection draws on normalised gates
        binding.sas_gate_normalize(s, logG, stream=stream)
        noisy_ms = time_noisy_select(w, logG, flush, stream, binding, device)
        del logG
        roofline["noisy_select_ms"] = round(noisy_ms, 4)
        roofline["noisy_select_gbs"] = round(noisy_select_bytes(w) / (noisy_ms * 1e-3) / 1e9, 1)
    res = {"workload": workload_desc(w), "value": round(job_throughput(step_flops, args.steps, total_ms, world), 3),
           "unit": "TFLOP/s", "ms_per_step": round(total_ms / args.steps, 4),
           "attended_gflop_per_step": round(step_flops / 1e9, 2), "gpu_launches": launches,
           "device_status": status, "roofline": roofline}
    return res, host


def run_gpu(args):
    from gated_block_sparse_flashattention_b200 import binding

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    w = workloads.WORKLOADS[args.workload]
    fwd_flops, bwd_flops = attended_flops(w)
    step_flops = fwd_flops + bwd_flops
    peaks = measured_peaks()
    stream = torch.cuda.current_stream(device)
    legs = set(args.legs.split(","))
    clk = ClockSampler(local).__enter__()   # running through every leg; samples kept while active
    time.sleep(0.3)
    clk.active = True

    head, host = None, None
    if "step" in legs:
        head, host = run_training(w, args, device, stream, binding, peaks, rank, world, noisy=True)
        torch.cuda.empty_cache()
    other = {}
    if "legs" in legs:
        for name in LEG_WORKLOADS:
            other[name], _ = run_training(workloads.WORKLOADS[name], args, device, stream, binding, peaks, rank,
                                          world)
            torch.cuda.empty_cache()

    # End to end through the C ABI from pinned host buffers, results copied back.
    if "e2e" in legs and host is None:
        host = rank_inputs(w, rank)
    e2e = run_e2e(args, w, host, device, stream, binding, step_flops, world) if "e2e" in legs else None
    host = None
    torch.cuda.empty_cache()
    dec = run_decode(args, device, stream, binding, peaks, clk) if "decode" in legs else None
    dec_paged = run_decode_paged(args, device, stream, binding, peaks, clk, args.paged_workload) \
        if "paged" in legs else None
    varlen = run_varlen(args, device, stream, binding, rank) if "varlen" in legs else None
    clk.active = False
    clk.__exit__(None, None, None)

    result = {
        "metric": METRIC,
        "value": head["value"] if head else None, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": head["ms_per_step"] if head else None, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": workload_desc(w), "global_batch": w.B * world, "seq_len": w.T,
                   "parallelism": f"dp{world} (replicas on independent batches)",
                   "l2": "flushed between timed steps (512 MiB write, outside the timed events)",
                   "attended_gflop_per_step": round(step_flops / 1e9, 2)},
        "roofline": head["roofline"] if head else None,
        "e2e": e2e,
        "gpu_launches": head["gpu_launches"] if head else 0,
        "device_status": head["device_status"] if head else None,
        "legs": other,
        "decode": dec,
        "decode_paged": dec_paged,
        "varlen": varlen,
    }
    if rank == 0 and world == 1 and "cpu" in legs:
        tf, threads, desc = oracle_sample(w, args.cpu_seconds)
        result["cpu_baseline"] = {"value": round(tf, 6), "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                                  "sample": desc}
    result["clocks"] = clk.summary()
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_varlen(args, device, stream, binding, rank):
    """The training step on a packed sequence: the Qwen3-4B-like layer's 8192 positions as five documents of
    512, 1536, 1024, 2048 and 3072 tokens (varlen gates and selection, then the unchanged forward, backward
    and selector gradient), device-resident inputs, L2 flushed between steps outside the events."""
    w = workloads.WORKLOADS[VARLEN_WORKLOAD]
    host = rank_inputs(w, rank)
    docs = VARLEN_DOCS
    cu = np.cumsum([0] + docs).tolist()
    Q, K, V, dO, s = (host[k].to(device) for k in ("Q", "K", "V", "dO", "s"))
    logG = torch.empty_like(s)
    tau = torch.empty(w.B, w.Hkv, w.T, device=device)
    tidx = torch.empty(w.B, w.Hkv, w.T, dtype=torch.int32, device=device)
    sel = torch.empty(w.B, w.Hkv, w.T, max(w.K - 1, 1), dtype=torch.int32, device=device)
    O, LSE = torch.empty_like(Q), torch.empty(w.B, w.Hq, w.T, device=device)
    dQ, dK, dV, dLogG, ds = (torch.empty_like(Q), torch.empty_like(K), torch.empty_like(V), torch.empty_like(s),
                             torch.empty_like(s))
    ws_f = binding.workspace(binding.sas_fwd_workspace_size(w.B, w.Hq, w.Hkv, w.T, w.d, w.K, 1), device)
    ws_b = binding.workspace(binding.sas_bwd_workspace_size(w.B, w.Hq, w.Hkv, w.T, w.d, w.K, 1), device)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)

    def step():
        binding.sas_gate_normalize_select_varlen(s, logG, tau, tidx, sel, w.K, cu, stream=stream)
        binding.sas_fwd(Q, K, V, logG, tau, tidx, O, LSE, w.K, w.sm_scale, ws_f, stream=stream, sel=sel)
        binding.sas_bwd(Q, K, V, O, dO, logG, tau, tidx, LSE, dQ, dK, dV, dLogG, w.K, w.sm_scale, ws_b,
                        stream=stream, sel=sel)
        binding.sas_gate_grad(logG, dLogG, ds, stream=stream)

    for _ in range(max(args.warmup, 3)):
        flush.zero_()
        step()
    torch.cuda.synchronize(device)
    times = []
    for _ in range(args.steps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        step()
        b.record(stream)
        times.append((a, b))
    torch.cuda.synchronize(device)
    ms = statistics.mean(a.elapsed_time(b) for a, b in times)
    fwd, bwd = attended_flops_varlen(w, docs)
    status = binding.sas_device_status(ws_f) or binding.sas_device_status(ws_b)
    return {"workload": f"{w.name} packed as documents of {docs} tokens", "ms_per_step": round(ms, 4),
            "value": round((fwd + bwd) / (ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
            "attended_gflop_per_step": round((fwd + bwd) / 1e9, 2), "device_status": status}


def run_e2e(args, w, host, device, stream, binding, step_flops, world):
    """The same step end to end from pinned host buffers through the library's calls: every step uploads its
    inputs (Q, K, V, dO, s) and downloads its outputs (O, dQ, dK, dV, ds). The steps are pipelined as a
    training loop feeding data from the host would run them: uploads on one stream, the step on another,
    downloads on a third, with two device buffers for the inputs and two for the outputs, so that the download
    of step i overlaps the upload of step i+1 and the step i+1 itself (the two copy directions run on separate
    copy engines). The timed region runs from before the first upload to after the last download of the timed
    steps; the inputs (2.4 GB) are larger than L2."""
    pinned = {k: host[k].pin_memory() for k in ("Q", "K", "V", "dO", "s")}
    out_host = {"O": torch.empty(host["Q"].shape, dtype=host["Q"].dtype).pin_memory(),
                "dQ": torch.empty(host["Q"].shape, dtype=host["Q"].dtype).pin_memory(),
                "dK": torch.empty(host["K"].shape, dtype=host["K"].dtype).pin_memory(),
                "dV": torch.empty(host["V"].shape, dtype=host["V"].dtype).pin_memory(),
                "ds": torch.empty(host["s"].shape, dtype=torch.float32).pin_memory()}
    dev_in = [{k: torch.empty(v.shape, dtype=v.dtype, device=device) for k, v in pinned.items()} for _ in range(2)]
    dev_out = [{k: torch.empty(v.shape, dtype=v.dtype, device=device) for k, v in out_host.items()}
               for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in pinned.values())
    d2h = sum(v.numel() * v.element_size() for v in out_host.values())
    # Step intermediates: the step stream runs one step at a time, so one set serves every step.
    gate_lse = torch.empty(w.B, w.Hkv, w.T, device=device)
    tau = torch.empty(w.B, w.Hkv, w.T, device=device)
    tidx = torch.empty(w.B, w.Hkv, w.T, dtype=torch.int32, device=device)
    sel = torch.empty(w.B, w.Hkv, w.T, max(w.K - 1, 1), dtype=torch.int32, device=device)
    LSE = torch.empty(w.B, w.Hq, w.T, device=device)
    dLogG = torch.empty(host["s"].shape, dtype=torch.float32, device=device)
    ws_f = binding.workspace(binding.sas_fwd_workspace_size(w.B, w.Hq, w.Hkv, w.T, w.d, w.K, 1), device)
    ws_b = binding.workspace(binding.sas_bwd_workspace_size(w.B, w.Hq, w.Hkv, w.T, w.d, w.K, 1), device)
    # Three non-blocking streams of their own (the default stream would serialise with them).
    s_in, s_cmp, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device), torch.cuda.Stream(device)
    for st_ in (s_in, s_cmp, s_out):
        st_.wait_stream(stream)   # the buffers above are allocated and zeroed on the caller's stream
    ev = lambda: torch.cuda.Event()  # noqa: E731
    in_ready, in_free, out_ready, out_free = ([ev(), ev()] for _ in range(4))

    def issue(i):
        b = i % 2
        x, y = dev_in[b], dev_out[b]
        if i >= 2:
            s_in.wait_event(in_free[b])
        with torch.cuda.stream(s_in):
            for k, v in pinned.items():
                x[k].copy_(v, non_blocking=True)
        in_ready[b].record(s_in)
        s_cmp.wait_event(in_ready[b])
        if i >= 2:
            s_cmp.wait_event(out_free[b])
        q, kk, vv, do, sc = x["Q"], x["K"], x["V"], x["dO"], x["s"]
        binding.sas_gate_normalize_select_compact(sc, gate_lse, tau, tidx, sel, w.K, stream=s_cmp)
        binding.sas_fwd(q, kk, vv, sc, tau, tidx, y["O"], LSE, w.K, w.sm_scale, ws_f, stream=s_cmp,
                        gate_lse=gate_lse, sel=sel)
        binding.sas_bwd(q, kk, vv, y["O"], do, sc, tau, tidx, LSE, y["dQ"], y["dK"], y["dV"], dLogG, w.K,
                        w.sm_scale, ws_b, stream=s_cmp, gate_lse=gate_lse, sel=sel)
        binding.sas_gate_grad(sc, dLogG, y["ds"], stream=s_cmp, gate_lse=gate_lse)
        in_free[b].record(s_cmp)
        out_ready[b].record(s_cmp)
        s_out.wait_event(out_ready[b])
        with torch.cuda.stream(s_out):
            for k, v in y.items():
                out_host[k].copy_(v, non_blocking=True)
        out_free[b].record(s_out)

    for i in range(max(1, args.warmup)):
        issue(i)
    torch.cuda.synchronize(device)
    barrier(device)
    a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(s_in)
    for i in range(args.steps):
        issue(i)
    e.record(s_out)
    e.synchronize()
    torch.cuda.synchronize(device)
    status = binding.sas_device_status(ws_f) or binding.sas_device_status(ws_b)
    if status:
        raise RuntimeError("kernel-side error in the end-to-end run")
    total = reduce_max(a.elapsed_time(e), device)
    return {"value": round(job_throughput(step_flops, args.steps, total, world), 3), "unit": "TFLOP/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(total / args.steps, 4),
            "pipeline": "uploads, step and downloads on three streams, double-buffered device inputs and outputs"}


def _time_decode_graph(call, n_rot, args, device, stream, binding, clk):
    """Captures n_rot back-to-back calls call(i) in one CUDA graph and returns the median device time per
    call (ms) over max(4, steps) replays, and the kernels one call launches."""
    g_stream = torch.cuda.Stream(device)
    g_stream.wait_stream(stream)
    launches0 = binding.launch_count()
    with torch.cuda.stream(g_stream):
        call(0, g_stream)
        per_call = binding.launch_count() - launches0
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=g_stream):
            for i in range(n_rot):
                call(i, g_stream)
    stream.wait_stream(g_stream)
    torch.cuda.synchronize(device)
    if clk is not None:
        clk.active = True
    for _ in range(max(args.warmup, 3)):
        graph.replay()
    torch.cuda.synchronize(device)
    reps = max(4, args.steps)
    times = []
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        graph.replay()
        b.record(stream)
        times.append((a, b))
    torch.cuda.synchronize(device)
    med = statistics.median([a.elapsed_time(b) for a, b in times]) / n_rot
    del graph
    return med, per_call, reps


def run_decode(args, device, stream, binding, peaks, clk=None):
    """Decode step (16 sequences x 1 token over a 32768-token cache), 16 steps per CUDA graph.

    The graph holds 16 decode steps back to back, each with its own seeded
    selector-score tensor, so every step attends a different random block set:
    one graph touches about 1 GB of distinct K/V blocks of the 2.1 GB cache, far
    more than the 126 MB L2, and a step's blocks come from HBM as in serving. The
    per-step time is the graph's device time / 16 (CUDA events around each
    replay), so host launch latency is amortised as it is in a decode loop.
    """
    w = workloads.WORKLOADS[DECODE_WORKLOAD]
    n_rot = 16
    inp = workloads.make_decode_inputs(w, seed=0)
    q, Kc, Vc = inp["q"].to(device), inp["Kc"].to(device), inp["Vc"].to(device)
    seqlen = inp["seqlen"].to(device)
    gen = torch.Generator().manual_seed(1)
    s_rot = [torch.randn(w.B, w.Hkv, w.NB, generator=gen).to(device) for _ in range(n_rot)]
    o = torch.empty_like(q)
    ws = binding.workspace(binding.sas_decode_workspace_size(w.B, w.Hq, w.Hkv, w.T, w.d, w.K), device)

    def call(i, st):
        binding.sas_decode_fwd(q, Kc, Vc, seqlen, s_rot[i], w.K, o, ws, w.sm_scale, stream=st)

    med, per_call, reps = _time_decode_graph(call, n_rot, args, device, stream, binding, clk)
    gbs = decode_bytes(w) / (med * 1e-3) / 1e9
    return {"workload": "decode_b16_l32k: 16 seqs x 1 token, cache 32768, Hq=32 Hkv=8 d=128 K=16",
            "value": round(gbs, 1), "unit": "GB/s", "us_per_step": round(med * 1e3, 2),
            "bytes_per_step": decode_bytes(w), "peak": peaks["hbm_gbs"],
            "frac": round(gbs / peaks["hbm_gbs"], 4), "traffic": measured_traffic("decode:" + DECODE_WORKLOAD),
            "graph": f"{n_rot} steps per graph", "steps": reps * n_rot,
            "launches_per_step": per_call, "device_status": binding.sas_device_status(ws),
            "l2": "not flushed; each step attends a different random block set (16 seeded score tensors)"}


def run_decode_paged(args, device, stream, binding, peaks, clk=None, name=PAGED_DECODE_WORKLOAD):
    """Long-context decode over a paged cache: 8 sequences x 1 token at 524288 tokens of context (8192 pages
    of 64 tokens per sequence, shuffled in a 19 GB pool), budget 32 blocks, 16 steps per CUDA graph with
    rotating seeded score tensors as in run_decode."""
    w = workloads.WORKLOADS[name]
    n_rot = 16
    inp = workloads.make_paged_decode_inputs(w, seed=0, device=device)
    gen = torch.Generator(device=device).manual_seed(1)
    s_rot = [torch.randn(w.B, w.Hkv, w.NB, generator=gen, device=device) for _ in range(n_rot)]
    o = torch.empty_like(inp["q"])
    ws = binding.workspace(binding.sas_decode_workspace_size(w.B, w.Hq, w.Hkv, w.T, w.d, w.K), device)

    def call(i, st):
        binding.sas_decode_fwd_paged(inp["q"], inp["Kp"], inp["Vp"], inp["page_table"], inp["seqlen"], s_rot[i],
                                     w.K, o, ws, w.sm_scale, stream=st)

    med, per_call, reps = _time_decode_graph(call, n_rot, args, device, stream, binding, clk)
    nbytes = decode_bytes(w) + w.B * w.Hkv * w.K * 4.0   # + the page-table entries of the attended blocks
    gbs = nbytes / (med * 1e-3) / 1e9
    pool_gb = 2 * inp["Kp"].numel() * inp["Kp"].element_size() / 1e9
    del inp
    return {"workload": f"{w.name}: {w.B} seqs x 1 token, context {w.T} ({w.NB} pages of 64 tokens "
                        f"each, {pool_gb:.1f} GB K/V pool), Hq={w.Hq} Hkv={w.Hkv} d={w.d} K={w.K}",
            "value": round(gbs, 1), "unit": "GB/s", "us_per_step": round(med * 1e3, 2),
            "bytes_per_step": nbytes, "peak": peaks["hbm_gbs"], "frac": round(gbs / peaks["hbm_gbs"], 4),
            "traffic": measured_traffic("decode_paged:" + name) if "decode_paged:" + name in MEASURED_TRAFFIC
            else None, "graph": f"{n_rot} steps per graph", "steps": reps * n_rot,
            "launches_per_step": per_call, "device_status": binding.sas_device_status(ws),
            "l2": "not flushed; each step attends a different random block set (16 seeded score tensors)"}


# ----------------------------------------------------------------------------- reference arm
def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return
    w = workloads.WORKLOADS[args.workload]
    per_step = max(2.0, args.cpu_seconds / max(1, args.steps))
    for _ in range(args.warmup):
        oracle_sample(w, 0.5)
    vals, threads, desc = [], 1, ""
    t0 = time.perf_counter()
    for _ in range(args.steps):
        v, threads, desc = oracle_sample(w, per_step)
        vals.append(v)
    wall = time.perf_counter() - t0
    value = statistics.mean(vals)
    print(json.dumps({
        "impl": "reference", "metric": METRIC,
        "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(wall / args.steps * 1e3, 1), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_desc(w)},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--workload", default=BENCH_WORKLOAD, choices=[BENCH_WORKLOAD, *LEG_WORKLOADS],
                    help="layer of the step leg (default: the headline layer; the others make smaller profiling runs)")
    ap.add_argument("--paged-workload", default=PAGED_DECODE_WORKLOAD,
                    choices=[PAGED_DECODE_WORKLOAD, "decode_b8_l64k_paged"],
                    help="paged decode leg (the 64K one keeps the pool at 2 GB for profiling runs)")
    ap.add_argument("--legs", default="step,legs,e2e,decode,paged,varlen,cpu",
                    help="comma list of what to measure and report: step (device-resident timed steps of the "
                         "headline layer), legs (the same step on the 8K and 64K layers), e2e (host buffers through "
                         "the C ABI), decode, paged (long-context paged decode), varlen (packed documents), cpu "
                         "(oracle baseline)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "native":
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
