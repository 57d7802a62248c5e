#!/usr/bin/env python
"""Benchmark of the B200 SSD library: prefill tokens/s (fraction of the bf16 tensor peak)
and cached decode steps/s (fraction of HBM bandwidth).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload prefill_2p7b_long|prefill_130m|decode_2p7b|...] [--no-extras]

One process per GPU (torchrun for N > 1).  Every rank runs its own independent
problem (weak scaling, no collective on the data path); rank 0 prints one JSON line
with the whole-job value = units of all ranks / max-over-ranks device time.

Workloads (synthetic, seeded; the shapes of Mamba-2 SSD layers):
  prefill_2p7b_long  bf16 x/B/C, fp32 dt/A/D/state: batch 4, 16384 tokens, 80 heads,
                     P 64, N 128, 1 group, chunk 256 (the largest single-GPU prefill: headline)
  prefill_130m       batch 8, 2048 tokens, 24 heads, P 64, N 128, chunk 256
  decode_2p7b        batch 64, 80 heads, P 64, N 128 fp32 state seeded by a 512-token
                     prefill; 1024 decode steps with fresh inputs, one CUDA graph
  deep_decode_2p7b   64 layers of that shape at batch 256 (42.9 GB of fp32 states), one token
                     per layer per step
The headline run also measures the other workloads and ends its JSON line with a short
"summary" of every workload's number.
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from state_space_model_05_b200 import inputs as gen  # noqa: E402

L2_BYTES = 126 * 2 ** 20
HEADLINE = "prefill_2p7b_long"
WORKLOADS = {
    "prefill_130m": dict(kind="prefill", batch=8, seqlen=2048, nheads=24, headdim=64, ngroups=1,
                         dstate=128, chunk_len=256, dtype="bf16"),
    "prefill_2p7b_long": dict(kind="prefill", batch=4, seqlen=16384, nheads=80, headdim=64,
                              ngroups=1, dstate=128, chunk_len=256, dtype="bf16"),
    "decode_2p7b": dict(kind="decode", batch=64, nheads=80, headdim=64, ngroups=1, dstate=128,
                        prefill_len=512, prefill_chunk=64, steps=1024, dtype="f32"),
    # Gated DeltaNet decode: the page's model shape (16 query/key heads, 32 value heads,
    # dk = dv = 128) at batch 1 (2 MB of state, L2-resident) and at batch 64 (128 MB, HBM)
    "gdn_decode_b1": dict(kind="gdn", batch=1, heads_qk=16, heads_v=32, dk=128, dv=128, steps=1024),
    "gdn_decode_b64": dict(kind="gdn", batch=64, heads_qk=16, heads_v=32, dk=128, dv=128, steps=256),
    "deep_decode_2p7b": dict(kind="deep_decode", layers=64, batch=256, nheads=80, headdim=64, ngroups=1,
                             dstate=128, steps=256, dtype="f32"),
    # ssd_decode_steps against one launch per step: the cached-decode shape, and batch 1
    # (where a launch per token costs more than the step's work)
    "decode_steps_2p7b": dict(kind="decode_steps", batch=64, nheads=80, headdim=64, ngroups=1, dstate=128,
                              steps=1024, dtype="f32"),
    "decode_steps_2p7b_b1": dict(kind="decode_steps", batch=1, nheads=80, headdim=64, ngroups=1, dstate=128,
                                 steps=1024, dtype="f32"),
    # ssd_decode_steps_layers: 64 layers of the 2.7B shape at batch 1 advanced by 64 tokens in
    # one launch, against one ssd_decode_step_layers launch per token (a CUDA graph)
    "decode_steps_stack_b1": dict(kind="decode_steps", layers=64, batch=1, nheads=80, headdim=64, ngroups=1,
                                  dstate=128, steps=64, dtype="f32"),
}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------------ accounting
TC_BLOCK = 128          # token block of the tensor-core path (a 256 chunk = two blocks)


def tc_path(w) -> bool:
    return w["dtype"] == "bf16" and w["headdim"] == 64 and w["dstate"] == 128 and w["chunk_len"] in (128, 256)


def prefill_flops(w, q=None) -> dict:
    """Algorithmic (causal-exact) FLOPs per call for chunk length q (default: the configured
    chunk), total and each kernel's share (the cumsum kernel does no tensor work)."""
    b, T, H, P, G, N = (w[k] for k in ("batch", "seqlen", "nheads", "headdim", "ngroups", "dstate"))
    Q = q or w["chunk_len"]
    tokens = b * T
    gemm1 = tokens * G * (Q + 1) * N          # C B^T, lower triangle incl. diagonal
    gemm2 = tokens * H * (Q + 1) * P          # (masked) X
    cstate = tokens * H * 2 * N * P           # chunk states
    cout = tokens * H * 2 * N * P             # carried state -> output
    return {"total": gemm1 + gemm2 + cstate + cout,
            "chunk_output_tc": gemm1 + gemm2 + cout, "chunk_output_simt": gemm1 + gemm2 + cout,
            "chunk_state_scan_tc": cstate, "chunk_state_simt": cstate,
            "block_gram_tc": gemm1, "chain_prefill_tc": gemm2 + cstate + cout}


def prefill_bytes(w) -> dict:
    """Algorithmic bytes per call: the whole path (x, dt, B, C read once, y and the final
    state written once), and per kernel of the tensor-core path, counting each kernel's
    own inputs and outputs once (the per-block state images and decay factors included)."""
    b, T, H, P, G, N, Q = (w[k] for k in ("batch", "seqlen", "nheads", "headdim", "ngroups", "dstate", "chunk_len"))
    e = 2 if w["dtype"] == "bf16" else 4
    c = -(-T // Q)
    io = b * T * (2 * H * P * e + 2 * G * N * e + H * 4) + b * H * P * N * 4
    nb = -(-T // TC_BLOCK)
    rows = b * H * nb * TC_BLOCK                 # (b, h, block, token) rows of the factor arrays
    image = b * H * nb * P * N * 2               # bf16 state at every block start
    return {"total": io,
            # dt in, fp16 copy of B (read bf16, write fp16), Lam/dt/two column-factor rows and
            # the chunk-state weights out
            "chunk_cumsum": b * T * H * 4 + 2 * b * T * G * N * 2 + 5 * rows * 4,
            # x, fp16 B and the weights in; block-start images and the final state out
            "chunk_state_scan_tc": b * T * (H * P * e + G * N * 2) + rows * 4 + image + b * H * P * N * 4,
            # x, B, C, block factors and block-start images in; y out
            "chunk_output_tc": b * T * (2 * H * P * e + 2 * G * N * e) + 4 * rows * 4 + image,
            "state_scan": 2 * b * H * c * P * N * 4 + b * H * P * N * 4,
            # fused path: B, C in; bf16 G = C B^T of every (b, g, block) out
            "block_gram_tc": 2 * b * T * G * N * e + b * G * nb * TC_BLOCK * TC_BLOCK * 2,
            # fused path: x, fp16 B, C, G and the block factors in; y and the final state out
            "chain_prefill_tc": b * T * (2 * H * P * e + 2 * G * N * 2) + b * G * nb * TC_BLOCK * TC_BLOCK * 2
                                + 4 * rows * 4 + b * H * P * N * 4}


def decode_bytes(w) -> int:
    b, H, P, G, N = (w[k] for k in ("batch", "nheads", "headdim", "ngroups", "dstate"))
    return 2 * b * H * P * N * 4 + 2 * b * H * P * 4 + 2 * b * G * N * 4 + b * H * 4


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def _code_only(text: str) -> str:
    """Source text without comments and with runs of whitespace collapsed: what the compiler
    sees, so that editing a comment does not discard a recorded measurement."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_source_sha() -> str:
    """Hash of every kernel source file (csrc and its subfolders): path and code, comments
    and layout excluded."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "state_space_model_05_b200", "csrc")
    files = []
    for dirpath, _, names in os.walk(csrc):
        files += [os.path.join(dirpath, n) for n in names if n.endswith((".cu", ".cuh", ".h"))]
    for path in sorted(files):
        with open(path, encoding="utf-8", errors="replace") as f:
            h.update((os.path.relpath(path, csrc) + "\0" + _code_only(f.read())).encode())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if taken on this source."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.txt")
    try:
        lines = open(path).read().splitlines()
    except OSError:
        return None
    sha = kernel_source_sha()
    for ln in lines:
        if ln.startswith("#") or "=" not in ln:
            continue
        kv = dict(tok.split("=", 1) for tok in ln.split())
        if kv.get("kernel") == kernel and kv.get("workload") == workload and kv.get("source_sha") == sha:
            return int(float(kv["dram_bytes_per_launch"]))
    return None


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi samples (200 ms) of this GPU's clocks and throttle reasons."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str | None):
        self.proc = None
        self.out = None
        if gpu_id is None:
            return
        try:
            self.out = open(f"/tmp/ssd_clocks_{os.getpid()}.csv", "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", gpu_id, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.out, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.close()
        rows = []
        for ln in open(self.out.name).read().splitlines():
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.out.name)
        if not rows:
            return {"samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------ distributed plumbing
def dist_setup():
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if torch.cuda.is_available():
        torch.cuda.set_device(local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def reduce_max(value: float, world: int) -> float:
    """Max over ranks of a host float (device time per rank)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def reduce_sum(value: float, world: int) -> float:
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def whole_job_rate(units_local: float, ms_local: float, world: int):
    """Weak scaling: every rank processed its own units in ms_local of device time.
    Returns (units of all ranks / max-over-ranks time in s, max-over-ranks ms)."""
    ms_max = reduce_max(ms_local, world)
    units = reduce_sum(units_local, world)
    return units / (ms_max / 1e3), ms_max


# ------------------------------------------------------------------ our arm
def _dev(a, dtype):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).to(device="cuda", dtype=dtype)


def prefill_problem(w, seed):
    shape = gen.SSDShape(w["batch"], w["seqlen"], w["nheads"], w["headdim"], w["ngroups"], w["dstate"])
    inp = gen.prefill_inputs(shape, seed=seed)
    if w["dtype"] == "bf16":
        inp.x, inp.B, inp.C = gen.round_bf16(inp.x), gen.round_bf16(inp.B), gen.round_bf16(inp.C)
    return inp


def run_prefill(w, steps, warmup, rank, world, name, e2e=True, dt_softplus=False):
    import torch
    import state_space_model_05_b200 as ssd
    from state_space_model_05_b200 import binding
    dt_ = torch.bfloat16 if w["dtype"] == "bf16" else torch.float32
    inp = prefill_problem(w, seed=rank)
    b, T, H, P, G, N, Q = (w[k] for k in ("batch", "seqlen", "nheads", "headdim", "ngroups", "dstate", "chunk_len"))
    code = binding.SSD_BF16 if w["dtype"] == "bf16" else binding.SSD_F32
    ws_bytes = ssd.ssd_prefill_workspace_bytes(b, T, H, P, G, N, Q, code)
    per_replica = prefill_bytes(w)["total"] + ws_bytes + b * T * H * P * (2 if w["dtype"] == "bf16" else 4)
    replicas = max(1, math.ceil(3 * L2_BYTES / per_replica))
    reps = []
    for _ in range(replicas):
        reps.append(dict(x=_dev(inp.x, dt_), dt=_dev(inp.dt_raw if dt_softplus else inp.dt, torch.float32),
                         dt_bias=_dev(inp.dt_bias, torch.float32), A=_dev(inp.A, torch.float32),
                         B=_dev(inp.B, dt_), C=_dev(inp.C, dt_), D=_dev(inp.D, torch.float32),
                         y=torch.empty((b, T, H, P), device="cuda", dtype=dt_),
                         st=torch.empty((b, H, P, N), device="cuda", dtype=torch.float32),
                         ws=torch.empty(ws_bytes, device="cuda", dtype=torch.uint8)))

    def step(i):
        r = reps[i % replicas]
        ssd.ssd_prefill(r["x"], r["dt"], r["A"], r["B"], r["C"], r["D"], Q, y=r["y"],
                        final_state=r["st"], workspace=r["ws"], dt_softplus=dt_softplus,
                        dt_bias=r["dt_bias"] if dt_softplus else None)

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    assert ssd.ssd_device_status() == 0
    # the timed region runs the calls back to back with no per-kernel events (an event
    # between two kernels would keep the dependent kernel from overlapping its setup with
    # the previous one's tail)
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    s0.record()
    for i in range(steps):
        step(i)
    s1.record()
    torch.cuda.synchronize()
    barrier(world)
    ms = s0.elapsed_time(s1)
    # per-kernel durations from a second pass with CUDA events around every launch
    prof_steps = min(steps, 50)
    binding.ssd_profile_reset()
    binding.ssd_profile_enable(True)
    for i in range(prof_steps):
        step(i)
    torch.cuda.synchronize()
    binding.ssd_profile_enable(False)
    kernels = binding.ssd_profile_read()
    status = ssd.ssd_device_status()
    if status != 0:
        raise RuntimeError(f"device status {status} after {name}")
    rate, ms_max = whole_job_rate(b * T * steps, ms, world)
    launches_per_step = sum(v[1] for v in kernels.values()) / prof_steps
    res = {"ms_total": ms_max, "ms_per_step": ms_max / steps, "tokens_per_s": rate,
           "kernels": kernels, "replicas": replicas, "launches": int(round(launches_per_step * steps))}

    if e2e:
        # end to end through the library's host-buffer entry (HostPrefill): every step copies
        # that step's inputs in from pinned host memory and y and the final state back out,
        # with step i's outputs travelling while step i + 1's inputs arrive and are computed
        from state_space_model_05_b200.host_pipeline import HostPrefill
        pin = lambda a, d: torch.from_numpy(np.ascontiguousarray(a)).to(d).pin_memory()
        hx, hdt, hB, hC = pin(inp.x, dt_), pin(inp.dt, torch.float32), pin(inp.B, dt_), pin(inp.C, dt_)
        outs = [(torch.empty((b, T, H, P), dtype=dt_).pin_memory(),
                 torch.empty((b, H, P, N), dtype=torch.float32).pin_memory()) for _ in range(2)]
        del reps
        torch.cuda.empty_cache()
        pipe = HostPrefill(b, T, H, P, G, N, Q, dt_, _dev(inp.A, torch.float32), _dev(inp.D, torch.float32))

        def e2e_run(n):
            for i in range(n):
                hy, hst = outs[i % 2]
                pipe.submit(hx, hdt, hB, hC, hy, hst)

        e2e_run(max(2, warmup))
        pipe.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(pipe.copy_in)
        e2e_run(steps)
        t1.record(pipe.copy_out)
        pipe.synchronize()
        torch.cuda.synchronize()
        barrier(world)
        erate, _ = whole_job_rate(b * T * steps, t0.elapsed_time(t1), world)
        h2d = sum(t.numel() * t.element_size() for t in (hx, hdt, hB, hC))
        hy, hst = outs[0]
        d2h = hy.numel() * hy.element_size() + hst.numel() * hst.element_size()
        res["e2e"] = {"value": erate, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                      "d2h_bytes_per_step": d2h,
                      "path": "HostPrefill: copies in and out overlapped with compute (two device buffer sets)"}
    return res


def varlen_lengths(total, seed=0, lo=64, hi=960):
    """Seeded sequence lengths, uniform in [lo, hi), cut to sum to ``total``."""
    rng = np.random.default_rng(seed)
    out = []
    while sum(out) < total:
        out.append(int(rng.integers(lo, hi)))
    out[-1] -= sum(out) - total
    return out


def run_prefill_varlen(w, steps, warmup, rank, world):
    """The prefill workload's tokens as one packed batch of mixed-length sequences."""
    import torch
    import state_space_model_05_b200 as ssd
    b, T, H, P, G, N, Q = (w[k] for k in ("batch", "seqlen", "nheads", "headdim", "ngroups", "dstate", "chunk_len"))
    total = b * T
    lengths = varlen_lengths(total, seed=rank)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32, device="cuda")
    inp = prefill_problem(dict(w, batch=1, seqlen=total), seed=rank)
    bf, f32 = torch.bfloat16, torch.float32
    per = total * (2 * H * P * 2 + 2 * G * N * 2 + H * 4) + 2 * len(lengths) * H * P * N * 4
    replicas = max(1, math.ceil(3 * L2_BYTES / per))
    reps = [dict(x=_dev(inp.x[0], bf), dt=_dev(inp.dt[0], f32), A=_dev(inp.A, f32), B=_dev(inp.B[0], bf),
                 C=_dev(inp.C[0], bf), D=_dev(inp.D, f32)) for _ in range(replicas)]
    for r in reps:
        r["y"], r["st"] = ssd.ssd_prefill_varlen(r["x"], r["dt"], r["A"], r["B"], r["C"], r["D"], cu, Q)
    nbytes = int(ssd.binding.lib().ssd_prefill_varlen_workspace_bytes(len(lengths), total, H, P, G, N, Q, 1))
    wsp = torch.empty(nbytes, device="cuda", dtype=torch.uint8)

    def step(i):
        r = reps[i % replicas]
        ssd.ssd_prefill_varlen(r["x"], r["dt"], r["A"], r["B"], r["C"], r["D"], cu, Q, y=r["y"],
                               final_states=r["st"], workspace=wsp)

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    s0.record()
    for i in range(steps):
        step(i)
    s1.record()
    torch.cuda.synchronize()
    barrier(world)
    if ssd.ssd_device_status() != 0:
        raise RuntimeError("device status after varlen prefill")
    rate, ms = whole_job_rate(total * steps, s0.elapsed_time(s1), world)
    return {"tokens_per_s": rate, "ms_per_step": ms / steps, "nseq": len(lengths),
            "lengths": f"{len(lengths)} sequences, {min(lengths)}..{max(lengths)} tokens (seeded)"}


def gdn_bytes(w) -> int:
    """Algorithmic bytes of one GDN decode step: the state read and written once, q, k, v,
    gate, beta read, the output written (fp32)."""
    b, hqk, hv, dk, dv = (w[k] for k in ("batch", "heads_qk", "heads_v", "dk", "dv"))
    return 2 * b * hv * dk * dv * 4 + 2 * b * hqk * dk * 4 + 2 * b * hv * dv * 4 + 2 * b * hv * 4


def run_gdn(w, repeats, warmup, rank, world):
    """GDN decode steps with per-step inputs pre-generated on the device, one CUDA graph
    of ``steps`` launches, timed with CUDA events over graph replays."""
    import torch
    import state_space_model_05_b200 as ssd
    shape = gen.GDNShape(w["batch"], w["heads_qk"], w["heads_v"], w["dk"], w["dv"])
    S = w["steps"]
    inp = gen.gdn_inputs(shape, S, seed=20 + rank)
    f32 = torch.float32
    Q, K, V, G, Bt = (_dev(a, f32) for a in (inp.q, inp.k, inp.v, inp.gate, inp.beta))
    state = _dev(inp.state, f32)
    out = torch.empty((shape.batch, shape.heads_v, shape.dv), device="cuda")
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for t in range(4):
            ssd.ssd_gdn_decode_step(state, Q[t], K[t], V[t], G[t], Bt[t], out=out)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            for t in range(S):
                ssd.ssd_gdn_decode_step(state, Q[t], K[t], V[t], G[t], Bt[t], out=out)
    for _ in range(warmup):
        graph.replay()
    torch.cuda.synchronize()
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    s0.record()
    for _ in range(repeats):
        graph.replay()
    s1.record()
    torch.cuda.synchronize()
    barrier(world)
    if ssd.ssd_device_status() != 0:
        raise RuntimeError("device status after GDN decode")
    steps_total = S * repeats
    rate, ms = whole_job_rate(steps_total, s0.elapsed_time(s1), world)
    nbytes = gdn_bytes(w)
    return {"steps_per_s": rate, "us_per_step": ms / steps_total * 1e3, "bytes_per_step": nbytes,
            "gbs": nbytes * steps_total / (ms / 1e3) / 1e9, "launches": steps_total}


def run_decode(w, repeats, warmup, rank, world):
    import torch
    import state_space_model_05_b200 as ssd
    from state_space_model_05_b200 import binding
    b, H, P, G, N, S = (w[k] for k in ("batch", "nheads", "headdim", "ngroups", "dstate", "steps"))
    shape = gen.SSDShape(b, w["prefill_len"], H, P, G, N)
    inp = gen.prefill_inputs(shape, seed=rank)
    f32 = torch.float32
    _, state = ssd.ssd_prefill(_dev(inp.x, f32), _dev(inp.dt, f32), _dev(inp.A, f32), _dev(inp.B, f32),
                               _dev(inp.C, f32), _dev(inp.D, f32), w["prefill_chunk"])
    dec = gen.decode_inputs(gen.SSDShape(b, 1, H, P, G, N), steps=S, seed=1000 + rank)
    X, DT, Bs, Cs = (_dev(a, f32) for a in (dec.x, dec.dt, dec.B, dec.C))
    A, D = _dev(inp.A, f32), _dev(inp.D, f32)
    y = torch.empty((b, H, P), device="cuda")
    del inp
    torch.cuda.synchronize()

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for k in range(4):                           # eager warm-up before capture
            ssd.ssd_decode_step(state, X[k], DT[k], A, Bs[k], Cs[k], D, y_t=y)
    torch.cuda.synchronize()

    def capture(profile: bool):
        binding.ssd_profile_reset()
        binding.ssd_profile_enable(profile)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.stream(side):
            with torch.cuda.graph(graph, stream=side):
                for k in range(S):
                    ssd.ssd_decode_step(state, X[k], DT[k], A, Bs[k], Cs[k], D, y_t=y)
        binding.ssd_profile_enable(False)
        return graph

    g = capture(False)                               # the timed loop: 1024 launches, no events
    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize()
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    s0.record()
    for _ in range(repeats):
        g.replay()
    s1.record()
    torch.cuda.synchronize()
    barrier(world)
    steps_total = S * repeats
    rate, ms = whole_job_rate(steps_total, s0.elapsed_time(s1), world)
    gp = capture(True)                               # same loop with an event pair per launch
    gp.replay()
    torch.cuda.synchronize()
    kernels = binding.ssd_profile_read()
    status = ssd.ssd_device_status()
    if status != 0:
        raise RuntimeError(f"device status {status} after decode")
    kms, klaunch = kernels.get("decode_step", (float("nan"), 0))
    nbytes = decode_bytes(w)
    res = {"steps_per_s": rate, "ms_per_step": ms / steps_total,
           "gbs": nbytes * steps_total / (ms / 1e3) / 1e9, "kernel_ms": kms / max(klaunch, 1),
           "launches": steps_total, "bytes_per_step": nbytes}
    del g, gp
    return res


def _timed_rate(fn, steps, repeats, warmup, world):
    """Steps/s of `fn` (one call = `steps` steps) over `repeats` calls, CUDA events, after
    `warmup` calls; max over ranks."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    e0.record()
    for _ in range(repeats):
        fn()
    e1.record()
    torch.cuda.synchronize()
    barrier(world)
    return whole_job_rate(steps * repeats, e0.elapsed_time(e1), world)


def run_decode_steps_stack(w, repeats, warmup, rank, world):
    """A stack of layers advanced by the workload's tokens two ways on the same
    device-resident per-layer inputs: one ssd_decode_step_layers launch per token (the whole
    stack, captured in a CUDA graph), and one ssd_decode_steps_layers launch for all tokens.
    Both compute the same result bit for bit."""
    import torch
    import state_space_model_05_b200 as ssd
    L, b, H, P, G, N, S = (w[k] for k in ("layers", "batch", "nheads", "headdim", "ngroups", "dstate", "steps"))
    shape = gen.SSDShape(b, 1, H, P, G, N)
    f32 = torch.float32
    layers = []
    for l in range(L):
        dec = gen.decode_inputs(shape, steps=S, seed=3000 + 10 * l + rank)
        A, D = gen.deep_head_params(l, H)
        X = _dev(dec.x, f32)
        layers.append(dict(state=_dev(gen.state_inputs(b, H, P, N, seed=3001 + 10 * l + rank), f32), x_t=X,
                           dt_t=_dev(dec.dt, f32), A=_dev(A, f32), B_t=_dev(dec.B, f32), C_t=_dev(dec.C, f32),
                           D=_dev(D, f32), y_t=torch.empty_like(X)))
    table = ssd.decode_layer_table(layers)
    per_token = [ssd.decode_layer_table([dict(ly, x_t=ly["x_t"][k], dt_t=ly["dt_t"][k], B_t=ly["B_t"][k],
                                              C_t=ly["C_t"][k], y_t=ly["y_t"][k]) for ly in layers])
                 for k in range(S)]
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for k in range(2):
            ssd.ssd_decode_step_layers(per_token[k], b, H, P, G, N, f32)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            for k in range(S):
                ssd.ssd_decode_step_layers(per_token[k], b, H, P, G, N, f32)
    per_step, _ = _timed_rate(graph.replay, S, repeats, warmup, world)
    one_launch, ms = _timed_rate(lambda: ssd.ssd_decode_steps_layers(table, S, b, H, P, G, N, f32), S, repeats,
                                 warmup, world)
    if ssd.ssd_device_status() != 0:
        raise RuntimeError("device status after stacked decode steps")
    del graph
    # one launch: every layer's state read and written once per call, its inputs and y once
    io = L * (S * (2 * b * H * P * 4 + 2 * b * G * N * 4 + b * H * 4) + 2 * b * H * P * N * 4)
    return {"steps_per_s_one_launch": one_launch, "steps_per_s_launch_per_step": per_step,
            "us_per_step_one_launch": ms / (S * repeats) * 1e3, "bytes_per_call": io,
            "gbs": io * repeats / (ms / 1e3) / 1e9}


def run_decode_steps(w, repeats, warmup, rank, world):
    """The decode workload's steps run two ways on the same device-resident inputs: one
    ssd_decode_step launch per token (captured in a CUDA graph), and one ssd_decode_steps
    launch for all of them.  Both compute the same result bit for bit.  A workload with
    several layers runs the stack version."""
    if w.get("layers", 1) > 1:
        return run_decode_steps_stack(w, repeats, warmup, rank, world)
    import torch
    import state_space_model_05_b200 as ssd
    b, H, P, G, N, S = (w[k] for k in ("batch", "nheads", "headdim", "ngroups", "dstate", "steps"))
    shape = gen.SSDShape(b, 1, H, P, G, N)
    dec = gen.decode_inputs(shape, steps=S, seed=2000 + rank)
    head = gen.prefill_inputs(shape, seed=2001 + rank)
    f32 = torch.float32
    X, DT, Bs, Cs = (_dev(a, f32) for a in (dec.x, dec.dt, dec.B, dec.C))
    A, D = _dev(head.A, f32), _dev(head.D, f32)
    state = _dev(gen.state_inputs(b, H, P, N, seed=2002 + rank), f32)
    Y = torch.empty((S, b, H, P), device="cuda")
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for k in range(4):
            ssd.ssd_decode_step(state, X[k], DT[k], A, Bs[k], Cs[k], D, y_t=Y[k])
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            for k in range(S):
                ssd.ssd_decode_step(state, X[k], DT[k], A, Bs[k], Cs[k], D, y_t=Y[k])

    def timed(fn):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize()
        e0.record()
        for _ in range(repeats):
            fn()
        e1.record()
        torch.cuda.synchronize()
        barrier(world)
        return whole_job_rate(S * repeats, e0.elapsed_time(e1), world)

    per_step, _ = timed(graph.replay)
    one_launch, ms = timed(lambda: ssd.ssd_decode_steps(state, X, DT, A, Bs, Cs, D, y=Y))
    if ssd.ssd_device_status() != 0:
        raise RuntimeError("device status after decode steps")
    del graph
    # one launch: the state is read and written once per call, the per-step inputs and y once
    io = S * (2 * b * H * P * 4 + 2 * b * G * N * 4 + b * H * 4) + 2 * b * H * P * N * 4
    return {"steps_per_s_one_launch": one_launch, "steps_per_s_launch_per_step": per_step,
            "us_per_step_one_launch": ms / (S * repeats) * 1e3, "bytes_per_call": io,
            "gbs": io * repeats / (ms / 1e3) / 1e9}


class DeepStack:
    """64 independent SSD layers of the 2.7B shape at batch 256: fp32 states (~43 GB) drawn
    i.i.d. N(0,1) on the device, and fresh per-layer inputs drawn on the device every step
    (counter-based generator; the host can regenerate any element)."""

    def __init__(self, w, one_launch=True):
        import torch
        self.w = w
        self.one_launch = one_launch
        L, b, H, P, G, N = (w[k] for k in ("layers", "batch", "nheads", "headdim", "ngroups", "dstate"))
        f32 = torch.float32
        self.states = torch.empty((L, b, H, P, N), device="cuda", dtype=f32)
        for l in range(L):
            gen.device_normal(self.states[l], gen.DEEP_SEED, gen.deep_stream(gen.DEEP_STATE, l))
        hp = [gen.deep_head_params(l, H) for l in range(L)]
        self.A = _dev(np.stack([a for a, _ in hp]), f32)
        self.D = _dev(np.stack([d for _, d in hp]), f32)
        self.x = torch.empty((L, b, H, P), device="cuda", dtype=f32)
        self.B = torch.empty((L, b, G, N), device="cuda", dtype=f32)
        self.C = torch.empty((L, b, G, N), device="cuda", dtype=f32)
        self.dt = torch.empty((L, b, H), device="cuda", dtype=f32)
        self.y = torch.empty((L, b, H, P), device="cuda", dtype=f32)
        self.table = _dev(gen.dt_table(), f32)
        self.inv = float(np.float32(1.0 / math.sqrt(N)))
        from state_space_model_05_b200 import binding
        self.layers = binding.decode_layer_table(
            [{"state": self.states[l], "x_t": self.x[l], "dt_t": self.dt[l], "A": self.A[l], "B_t": self.B[l],
              "C_t": self.C[l], "D": self.D[l], "y_t": self.y[l]} for l in range(L)])

    def draw(self, step):
        for l in range(self.w["layers"]):
            gen.device_normal(self.x[l], gen.DEEP_SEED, gen.deep_stream(gen.DEEP_X, l, step))
            gen.device_normal(self.B[l], gen.DEEP_SEED, gen.deep_stream(gen.DEEP_B, l, step), self.inv)
            gen.device_normal(self.C[l], gen.DEEP_SEED, gen.deep_stream(gen.DEEP_C, l, step), self.inv)
            gen.device_table(self.dt[l], self.table, gen.DT_TABLE_BITS, gen.DEEP_SEED,
                             gen.deep_stream(gen.DEEP_DT, l, step))

    def step(self):
        """One token for every layer: one launch for the whole stack, or one per layer."""
        import state_space_model_05_b200 as ssd
        w = self.w
        if self.one_launch:
            ssd.ssd_decode_step_layers(self.layers, w["batch"], w["nheads"], w["headdim"], w["ngroups"],
                                       w["dstate"], self.x.dtype)
            return
        for l in range(w["layers"]):
            ssd.ssd_decode_step(self.states[l], self.x[l], self.dt[l], self.A[l], self.B[l], self.C[l],
                                self.D[l], y_t=self.y[l])


def run_deep_decode(w, steps, warmup, rank, world, one_launch=True):
    """Per step: draw the step's inputs (untimed), then time the decode of all L layers
    (one launch for the stack, or one launch per layer)."""
    import torch
    import state_space_model_05_b200 as ssd
    stack = DeepStack(w, one_launch=one_launch)
    steps = min(steps, w["steps"])
    for k in range(warmup):                         # warm-up steps use their own streams
        stack.draw(w["steps"] + k)
        stack.step()
    torch.cuda.synchronize()
    evs = []
    barrier(world)
    for k in range(steps):
        stack.draw(k)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        stack.step()
        e1.record()
        evs.append((e0, e1))
    torch.cuda.synchronize()
    barrier(world)
    ms_local = sum(a.elapsed_time(b) for a, b in evs)
    if ssd.ssd_device_status() != 0:
        raise RuntimeError("device status after deep decode")
    rate, ms = whole_job_rate(steps, ms_local, world)
    L, b, H, P, G, N = (w[k] for k in ("layers", "batch", "nheads", "headdim", "ngroups", "dstate"))
    per_layer = decode_bytes({"batch": b, "nheads": H, "headdim": P, "ngroups": G, "dstate": N})
    res = {"steps_per_s": rate, "ms_per_step": ms / steps, "bytes_per_step": L * per_layer,
           "gbs": L * per_layer * steps / (ms / 1e3) / 1e9, "launches": steps * (1 if one_launch else L),
           "steps": steps}
    del stack
    torch.cuda.empty_cache()
    return res


def roofline_prefill(w, res, peaks, src, workload):
    """Roofline of the dominant kernel against the bf16 tensor peak: its share of the
    chunked method's algorithmic (causal-exact) FLOPs per launch over its average launch
    duration.  Beside it: the whole path's algorithmic bytes (x, dt, B and C read once, y
    and the final state written once), the kernel's own design traffic, and the DRAM bytes
    ncu measured for that kernel (null unless taken on the current sources)."""
    kernels = res["kernels"]
    dom = max(kernels, key=lambda k: kernels[k][0])
    ms, n = kernels[dom]
    per_launch_ms = ms / n
    flops = prefill_flops(w).get(dom, 0)
    achieved = flops / (per_launch_ms / 1e3) / 1e12
    peak = peaks["bf16_tflops"]
    design = prefill_bytes(w).get(dom)
    traffic = recorded_traffic(dom, workload)
    algo = prefill_bytes(w)["total"]
    return {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
            "traffic": traffic, "kernel": dom, "kernel_ms": per_launch_ms, "kernel_flops": flops,
            "frac_of_sustained": achieved / peaks.get("bf16_tflops_sustained", peak),
            "algorithmic_bytes": algo, "design_bytes": design,
            "traffic_over_algorithmic": (traffic / algo) if traffic else None,
            "peak_source": src, "peak_note": "burst cuBLAS bf16 (the kernel runs in a short timed region)"}


def prefill_entry(w, workload, res, peaks, src):
    """The numbers of one prefill workload (headline or extra)."""
    sec = res["ms_per_step"] / 1e3
    flops = prefill_flops(w)["total"]
    out = {"value": res["tokens_per_s"], "unit": "tokens/s", "ms_per_step": res["ms_per_step"],
           "prefill_tflops": flops / sec / 1e12, "prefill_tensor_frac": flops / sec / 1e12 / peaks["bf16_tflops"],
           "prefill_hbm_gbs": prefill_bytes(w)["total"] / sec / 1e9,
           "prefill_hbm_frac": prefill_bytes(w)["total"] / sec / 1e9 / peaks["hbm_gbs"],
           "roofline": roofline_prefill(w, res, peaks, src, workload),
           "kernels_ms": {k: v[0] / v[1] for k, v in res["kernels"].items()}}
    if tc_path(w):
        out["prefill_tflops_executed"] = prefill_flops(w, TC_BLOCK)["total"] / sec / 1e12
    return out


def decode_roofline(gbs, kernel, peaks, src, traffic=None):
    return {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"],
            "traffic": traffic, "kernel": kernel, "peak_source": src}


def ours(args, rank, world):
    import torch
    from state_space_model_05_b200.build import build
    build()
    w = WORKLOADS[args.workload]
    peaks, src = load_peaks()
    from state_space_model_05_b200 import binding as _binding
    _binding.ssd_set_prefill_path(args.prefill_path)
    gpu_id = None
    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(torch.cuda.current_device()).uuid)
    except Exception:  # noqa: BLE001
        gpu_id = str(torch.cuda.current_device())
    clocks = ClockSampler(gpu_id)
    line = {"metric": "", "value": None, "unit": "", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": None, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "data": "synthetic (seeded generators, state_space_model_05_b200/inputs.py)"}
    summary = {}
    solo = rank == 0 and world == 1 and not args.no_cpu_baseline
    if w["kind"] == "prefill":
        res = run_prefill(w, args.steps, args.warmup, rank, world, args.workload)
        entry = prefill_entry(w, args.workload, res, peaks, src)
        line.update({"metric": "SSD prefill tokens/s", "value": res["tokens_per_s"], "unit": "tokens/s",
                     "ms_per_step": res["ms_per_step"], "dtype": w["dtype"]})
        line["roofline"] = entry.pop("roofline")
        for k in ("prefill_tflops", "prefill_tensor_frac", "prefill_tflops_executed", "prefill_hbm_gbs",
                  "prefill_hbm_frac", "kernels_ms"):
            if k in entry:
                line[k] = entry[k]
        line["e2e"] = res.get("e2e")
        line["gpu_launches"] = res["launches"]
        cfg = {"workload": args.workload, **{k: w[k] for k in w if k != "kind"},
               "l2": f"inputs rotated over {res['replicas']} resident replicas (> 3x L2) between steps"}
        summary[args.workload] = {"tok_s": round(res["tokens_per_s"]), "ms": round(res["ms_per_step"], 4),
                                  "tensor_frac": round(line["prefill_tensor_frac"], 4),
                                  "kernel_frac": round(line["roofline"]["frac"], 4)}
    elif w["kind"] == "gdn":
        res = run_gdn(w, max(1, args.steps // 100), max(1, args.warmup // 3), rank, world)
        line.update({"metric": "GDN decode steps/s", "value": res["steps_per_s"], "unit": "steps/s",
                     "ms_per_step": res["us_per_step"] / 1e3, "dtype": "f32"})
        line["roofline"] = decode_roofline(res["gbs"], "gdn_decode_step", peaks, src)
        line["gpu_launches"] = res["launches"]
        line["e2e"] = None
        cfg = {"workload": args.workload, **{k: w[k] for k in w if k != "kind"}}
    elif w["kind"] == "decode_steps":
        res = run_decode_steps(w, max(1, args.steps // 4), max(1, args.warmup), rank, world)
        line.update({"metric": "SSD decode steps/s (all steps in one launch)", "value": res["steps_per_s_one_launch"],
                     "unit": "steps/s", "ms_per_step": res["us_per_step_one_launch"] / 1e3, "dtype": "f32"})
        line["roofline"] = decode_roofline(res["gbs"], "decode_steps", peaks, src,
                                           recorded_traffic("decode_steps", args.workload))
        line["launch_per_step_steps_per_s"] = res["steps_per_s_launch_per_step"]
        line["gpu_launches"] = max(1, args.steps // 4)
        line["e2e"] = None
        cfg = {"workload": args.workload, **{k: w[k] for k in w if k != "kind"}}
        if solo:
            line["cpu_baseline"] = cpu_baseline_decode(w, budget_s=8.0)
    elif w["kind"] == "deep_decode":
        res = run_deep_decode(w, args.steps, 3, rank, world)
        line.update({"metric": "SSD decode steps/s (64-layer stack)", "value": res["steps_per_s"],
                     "unit": "steps/s", "ms_per_step": res["ms_per_step"], "dtype": "f32"})
        line["roofline"] = decode_roofline(res["gbs"], "decode_layers (all layers, one launch per step)", peaks, src)
        line["gpu_launches"] = res["launches"]
        line["e2e"] = None
        cfg = {"workload": args.workload, **{k: w[k] for k in w if k != "kind"}}
        if solo:
            line["cpu_baseline"] = cpu_baseline_decode(w, budget_s=8.0)
    else:
        res = run_decode(w, max(1, args.steps // 100), max(1, args.warmup // 3), rank, world)
        line.update({"metric": "SSD decode steps/s", "value": res["steps_per_s"], "unit": "steps/s",
                     "ms_per_step": res["ms_per_step"], "dtype": "f32"})
        kgbs = res["bytes_per_step"] / (res["ms_per_step"] / 1e3) / 1e9
        line["roofline"] = decode_roofline(kgbs, "decode_step", peaks, src,
                                           recorded_traffic("decode_step", args.workload))
        line["gpu_launches"] = res["launches"]
        line["e2e"] = None
        cfg = {"workload": args.workload, **{k: w[k] for k in w if k != "kind"}}
        if solo:
            line["cpu_baseline"] = cpu_baseline_decode(w, budget_s=8.0)
    cfg["parallelism"] = f"independent problem per GPU x{world}"
    if args.prefill_path != "auto":
        cfg["prefill_path"] = args.prefill_path
    line["config"] = cfg

    if not args.no_extras and args.workload == HEADLINE:
        extras = {}
        # the 130M-shaped layer (the other prefill configuration), on the default path
        pw = WORKLOADS["prefill_130m"]
        r = run_prefill(pw, 100, 5, rank, world, "prefill_130m", e2e=False)
        e = prefill_entry(pw, "prefill_130m", r, peaks, src)
        e["config"] = {k: pw[k] for k in pw if k != "kind"}
        extras["prefill_130m"] = e
        summary["prefill_130m"] = {"tok_s": round(r["tokens_per_s"]), "ms": round(r["ms_per_step"], 4),
                                   "tensor_frac": round(e["prefill_tensor_frac"], 4),
                                   "kernel_frac": round(e["roofline"]["frac"], 4)}
        # both prefill workloads on each tensor-core path, for comparison with the default
        for path in ("fused", "two_pass"):
            prev_path = _binding.ssd_set_prefill_path(path)
            try:
                for name in (args.workload, "prefill_130m"):
                    pw2 = WORKLOADS[name]
                    r = run_prefill(pw2, 20 if name == args.workload else 100, 3, rank, world, f"{name}_{path}", e2e=False)
                    extras[f"{name}_{path}_path"] = {"value": r["tokens_per_s"], "unit": "tokens/s",
                                                     "ms_per_step": r["ms_per_step"],
                                                     "kernels_ms": {k: v[0] / v[1] for k, v in r["kernels"].items()}}
                    summary[f"{name}_{path}"] = {"tok_s": round(r["tokens_per_s"]), "ms": round(r["ms_per_step"], 4)}
            finally:
                _binding.ssd_set_prefill_path(prev_path)
        # cached decode: 1024 steps in one CUDA graph; every launch in the timed graph is a
        # decode kernel, so the average launch duration is the timed region over the launches
        dw = WORKLOADS["decode_2p7b"]
        d = run_decode(dw, 3, 1, rank, world)
        kgbs = d["bytes_per_step"] / (d["ms_per_step"] / 1e3) / 1e9
        extras["decode_2p7b"] = {"value": d["steps_per_s"], "unit": "steps/s", "ms_per_step": d["ms_per_step"],
                                 "kernel_ms_event_pairs": d["kernel_ms"],
                                 "roofline": decode_roofline(kgbs, "decode_step", peaks, src,
                                                             recorded_traffic("decode_step", "decode_2p7b")),
                                 "config": {k: dw[k] for k in dw if k != "kind"}}
        summary["decode_2p7b"] = {"steps_s": round(d["steps_per_s"]), "us": round(d["ms_per_step"] * 1e3, 2),
                                  "hbm_frac": round(kgbs / peaks["hbm_gbs"], 4)}
        ddw = WORKLOADS["deep_decode_2p7b"]
        dd = run_deep_decode(ddw, 64, 3, rank, world, one_launch=True)
        dp = run_deep_decode(ddw, 16, 3, rank, world, one_launch=False)
        extras["deep_decode_2p7b"] = {"value": dd["steps_per_s"], "unit": "steps/s", "ms_per_step": dd["ms_per_step"],
                                      "steps_timed": dd["steps"], "launches_per_step": 1,
                                      "roofline": decode_roofline(dd["gbs"], "decode_layers (64 layers, one launch)",
                                                                  peaks, src),
                                      "per_layer_launches": {"value": dp["steps_per_s"], "ms_per_step": dp["ms_per_step"],
                                                             "gbs": dp["gbs"], "launches_per_step": ddw["layers"]},
                                      "config": {k: ddw[k] for k in ddw if k != "kind"}}
        summary["deep_decode_2p7b"] = {"steps_s": round(dd["steps_per_s"], 2), "ms": round(dd["ms_per_step"], 3),
                                       "hbm_frac": round(dd["gbs"] / peaks["hbm_gbs"], 4)}
        # the headline prefill with dt = softplus(dt_raw + dt_bias) formed in the kernels
        r = run_prefill(pw, 100, 5, rank, world, "prefill_130m_dtraw", e2e=False, dt_softplus=True)
        extras["prefill_130m_dt_softplus"] = {"value": r["tokens_per_s"], "unit": "tokens/s",
                                              "ms_per_step": r["ms_per_step"]}
        # the 130M workload's tokens as one packed batch of mixed-length sequences
        vr = run_prefill_varlen(pw, 100, 5, rank, world)
        extras["prefill_130m_varlen"] = {"value": vr["tokens_per_s"], "unit": "tokens/s",
                                         "ms_per_step": vr["ms_per_step"], "sequences": vr["lengths"]}
        for name in ("decode_steps_2p7b", "decode_steps_2p7b_b1", "decode_steps_stack_b1"):
            sw = WORKLOADS[name]
            r = run_decode_steps(sw, 5, 2, rank, world)
            extras[name] = {"value": r["steps_per_s_one_launch"], "unit": "steps/s",
                            "us_per_step": r["us_per_step_one_launch"],
                            "launch_per_step_steps_per_s": r["steps_per_s_launch_per_step"],
                            "roofline": decode_roofline(r["gbs"], "decode_steps (all steps, one launch; state "
                                                        "read and written once per call)", peaks, src,
                                                        recorded_traffic("decode_steps", name)),
                            "config": {k: sw[k] for k in sw if k != "kind"}}
            summary[name] = {"steps_s": round(r["steps_per_s_one_launch"]),
                             "launch_per_step_steps_s": round(r["steps_per_s_launch_per_step"])}
        for name in ("gdn_decode_b1", "gdn_decode_b64"):
            gw = WORKLOADS[name]
            r = run_gdn(gw, 3, 1, rank, world)
            extras[name] = {"value": r["steps_per_s"], "unit": "steps/s", "us_per_step": r["us_per_step"],
                            "roofline": dict(decode_roofline(r["gbs"], "gdn_decode_step", peaks, src),
                                             note="state L2-resident" if gw["batch"] == 1 else "state in HBM"),
                            "config": {k: gw[k] for k in gw if k != "kind"}}
            summary[name] = {"steps_s": round(r["steps_per_s"]), "us": round(r["us_per_step"], 2),
                             "hbm_frac": round(r["gbs"] / peaks["hbm_gbs"], 4)}
        if solo:
            extras["prefill_130m"]["cpu_baseline"] = cpu_baseline(pw, budget_s=6.0)
            extras["decode_2p7b"]["cpu_baseline"] = cpu_baseline_decode(dw, budget_s=6.0)
            extras["deep_decode_2p7b"]["cpu_baseline"] = cpu_baseline_decode(ddw, budget_s=6.0)
        line.update(extras)
    line["clocks"] = clocks.stop()
    if solo and w["kind"] == "prefill":
        line["cpu_baseline"] = cpu_baseline(w, budget_s=20.0)
    # last, so that a reader of the end of the output sees every workload's number
    line["summary"] = summary
    return line


# ------------------------------------------------------------------ oracle timing
def host_cores() -> int:
    """The host cores this process may run on (the oracle's all-core runs use them all; the
    thread count is passed on every call, since an OpenMP thread-count setting persists)."""
    try:
        return len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        return os.cpu_count() or 1


def oracle_sample_step(w, inp, units, nthreads=0):
    import oracle
    t = time.perf_counter()
    oracle.prefill(inp.x, inp.dt, inp.A, inp.B, inp.C, inp.D, units=units, nthreads=nthreads or host_cores())
    return time.perf_counter() - t


def cpu_baseline(w, budget_s=20.0):
    """The fp64 oracle on a bounded sample of the prefill workload's (batch, head) units, on
    all host cores, and on one core for one unit."""
    import oracle
    oracle.build()
    inp = prefill_problem(w, seed=0)
    H, T = w["nheads"], w["seqlen"]
    n_all = w["batch"] * H
    probe = list(range(min(n_all, host_cores())))
    t1 = oracle_sample_step(w, inp, probe)
    per_unit = t1 / len(probe)
    n = int(min(n_all, max(len(probe), budget_s / max(per_unit, 1e-9))))
    units = list(range(n))
    t = oracle_sample_step(w, inp, units)
    t_one = oracle_sample_step(w, inp, [0], nthreads=1)
    tokens = n / H * T
    return {"value": tokens / t, "unit": "tokens/s", "cores": host_cores(), "kind": "oracle",
            "single_core": {"value": T / H / t_one, "unit": "tokens/s", "cores": 1},
            "sample": f"{n} of {n_all} (batch, head) units of the {w['batch']}x{T}-token workload, "
                      f"fp64 sequential recurrence, {t:.2f} s; one unit on one core, {t_one:.2f} s"}


def _decode_units(w):
    """(units per step, batch, heads) of a decode workload (a unit is one (layer, b, h))."""
    layers = w.get("layers", 1)
    return layers * w["batch"] * w["nheads"], w["batch"], w["nheads"]


def oracle_decode_rate(w, budget_s, nthreads=0, seed=0):
    """Decode steps/s of the fp64 oracle: steps of a sample of units (one layer's batch and
    heads), scaled to the workload's units per step."""
    import oracle
    oracle.build()
    per_step, b, H = _decode_units(w)
    P, G, N = w["headdim"], w["ngroups"], w["dstate"]
    shape = gen.SSDShape(b, 1, H, P, G, N)
    dec = gen.decode_inputs(shape, steps=4, seed=seed + 7)
    hp = gen.prefill_inputs(gen.SSDShape(1, 1, H, P, G, N), seed=seed)
    n_all = b * H
    cores = nthreads or host_cores()
    units = list(range(min(n_all, max(64, 64 * cores))))
    state = gen.state_inputs(1, len(units), P, N, seed=seed + 8)[0].astype(np.float64)
    t0, steps = time.perf_counter(), 0
    while True:
        k = steps % 4
        oracle.decode_step(state, dec.x[k], dec.dt[k], hp.A, dec.B[k], dec.C[k], hp.D, units=units, nthreads=cores)
        steps += 1
        el = time.perf_counter() - t0
        if el >= budget_s or steps >= 4096:
            break
    unit_steps_per_s = len(units) * steps / el
    return unit_steps_per_s / per_step, len(units), steps, el, cores


def cpu_baseline_decode(w, budget_s=6.0):
    rate, nu, st, el, cores = oracle_decode_rate(w, budget_s)
    one, nu1, st1, el1, _ = oracle_decode_rate(w, max(1.0, budget_s / 4), nthreads=1)
    per_step, _, _ = _decode_units(w)
    return {"value": rate, "unit": "steps/s", "cores": cores, "kind": "oracle",
            "single_core": {"value": one, "unit": "steps/s", "cores": 1},
            "sample": f"{st} steps of {nu} of the {per_step} (layer, batch, head) units a step, fp64, "
                      f"{el:.2f} s, scaled to whole steps; one core: {st1} steps of {nu1} units, {el1:.2f} s"}


def reference(args, rank, world):
    """The fp64 CPU oracle as the reference arm (rank 0 only)."""
    import oracle
    oracle.build()
    w = WORKLOADS[args.workload]
    cfg = {"workload": args.workload, **{k: w[k] for k in w if k != "kind"}}
    base = {"impl": "reference", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded)", "config": cfg}
    if w["kind"] in ("decode", "deep_decode", "decode_steps"):
        budget = 150.0 / max(1, args.steps + args.warmup)
        for _ in range(args.warmup):
            oracle_decode_rate(w, budget / 4)
        rates = [oracle_decode_rate(w, budget) for _ in range(args.steps)]
        value = statistics.mean(r[0] for r in rates)
        nu, st = rates[0][1], rates[0][2]
        per_step, _, _ = _decode_units(w)
        sample = f"each step: {st} decode steps of {nu} of the {per_step} units a step, scaled to whole steps"
        metric = {"decode": "SSD decode steps/s", "deep_decode": "SSD decode steps/s (64-layer stack)",
                  "decode_steps": "SSD decode steps/s (all steps in one launch)"}[w["kind"]]
        return dict(base, metric=metric, value=value, unit="steps/s", ms_per_step=1e3 / value,
                    cpu_baseline={"value": value, "unit": "steps/s", "cores": host_cores(), "kind": "oracle",
                                  "sample": sample},
                    e2e={"value": value, "unit": "steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0})
    if w["kind"] != "prefill":
        return {"impl": "reference", "unavailable": "the oracle reference arm times the SSD prefill and decode workloads"}
    inp = prefill_problem(w, seed=0)
    H, T = w["nheads"], w["seqlen"]
    n_all = w["batch"] * H
    probe = list(range(min(n_all, host_cores())))
    per_unit = oracle_sample_step(w, inp, probe) / len(probe)
    budget = 150.0 / max(1, args.steps + args.warmup)
    n = int(min(n_all, max(len(probe), budget / max(per_unit, 1e-9))))
    units = list(range(n))
    for _ in range(args.warmup):
        oracle_sample_step(w, inp, units)
    total = sum(oracle_sample_step(w, inp, units) for _ in range(args.steps))
    tokens = n / H * T * args.steps
    value = tokens / total
    sample = f"{n} of {n_all} (batch, head) units per step of the {w['batch']}x{T}-token workload"
    return dict(base, metric="SSD prefill tokens/s", value=value, unit="tokens/s",
                ms_per_step=total / args.steps * 1e3,
                cpu_baseline={"value": value, "unit": "tokens/s", "cores": host_cores(), "kind": "oracle",
                              "sample": sample},
                e2e={"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0})


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default=HEADLINE)
    ap.add_argument("--no-extras", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--prefill-path", choices=["auto", "fused", "two_pass"], default="auto",
                    help="tensor-core prefill kernels (ssd_set_prefill_path)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        if rank != 0:
            return 0
        print(json.dumps(reference(args, rank, world)), flush=True)
        return 0
    rank, world, _ = dist_setup()
    try:
        line = ours(args, rank, world)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
