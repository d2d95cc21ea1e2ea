"""Throughput of the DSA hot path on B200: query-tokens/s of one step = lightning indexer ->
top-k -> sparse MLA (and, for the sparse-stage workload, p emission + indexer KL) over one
batch of seeded synthetic inputs, plus each stage's roofline fraction.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl dsa|reference]
                  [--scaling weak|strong] [--no-extra] [--peaks] [--dry-run]

Default workload: long_prefill_32k (B=1, L=32768 causal, the largest single-GPU workload). With
N = 1 the same JSON line also carries a `decode_128k` block (the 128K-context decode, B=32 queries
against 131072 keys each) and a `workloads` block with every other workload, each timed the same
way with fewer steps.

N > 1: `--gpus N` re-launches itself under torch.distributed.run, one rank per GPU (NCCL).
  weak (default): the job is N copies of the workload's batch (N*B sequences drawn from the
    seeded streams); each rank takes its sequences with shard_rows, so per-GPU work is fixed.
  strong: the workload's batch is fixed; decode rows are split with shard_rows and causal
    prefill rows with shard_causal_rows (rank r computes query rows [start, stop) against keys
    [0, stop)).
The sparse-stage loss is summed over ranks (one NCCL all-reduce per step, the path's only
collective); step time is the max over ranks.  `--dry-run` stops before CUDA: every rank (gloo)
reports its shard and rank 0 prints them, so the launcher and the sharding are testable on CPU.

`--impl reference` times the fp64 CPU oracle on a bounded sample of the same workload.
`--peaks` measures the FP8 and bf16 dense GEMM peaks (torch._scaled_mm / torch.matmul, 8192^3)
and a read-only HBM reference (torch.sum over 1 GiB and 4 GiB) with CUDA events.
Prints ONE JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import socket
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import dsa_inputs  # noqa: E402
from sparse_attention_tcgen05_b200.sharding import (MLA_WEIGHT, max_over_ranks,  # noqa: E402
                                                    shard_causal_rows, shard_rows, sum_over_ranks)

METRIC = "query-tokens/s (indexer+top-k+sparse MLA) at 1 B200; % of roofline per stage"
DEFAULT_WORKLOAD = "long_prefill_32k"
DECODE_TARGET = "decode_128k"  # the decode workload held to a path-roofline target
L2_FLUSH_BYTES = 512 << 20
# FP8 e4m3 dense rate relative to bf16 (NVIDIA B200 datasheet, dense: 4.5 vs 2.25 PFLOP/s)
FP8_OVER_BF16 = 2.0


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


# ---------------------------------------------------------------------------------- work model
def algorithmic(wl):
    """Algorithmic bytes and MACs per step of each stage: causal pairs and selected entries only.
    indexer: reads k_I, q_I, w once and writes the [B,Lq,Lk] scores; MACs over visible pairs.
    top-k: reads the visible scores once, writes idx.  sparse MLA: reads q, idx and the unique
    latent rows it selects once, writes out and lse; MACs = selected x H x (d_qk + d_v)."""
    B, Lq, Lk, k = wl.B, wl.Lq, wl.Lk, wl.k
    t = np.arange(Lq) + (Lk - Lq)
    vis = (t + 1).astype(np.float64)            # visible keys per query
    if wl.dense:
        # the dense warm-up step: indexer, dense attention (lse pass, p pass, output) with the
        # target p written for every (t, s), eq. (3) over every visible pair
        pairs = B * vis.sum()
        ix = {"bytes": B * Lk * wl.d_I + B * Lq * wl.H_I * (wl.d_I + 4) + B * Lq * Lk * 4,
              "macs": pairs * wl.H_I * wl.d_I}
        dm = {"bytes": 2 * B * Lq * wl.H * wl.d_qk + 2 * B * Lk * wl.d_qk + 2 * B * Lq * wl.H * wl.d_v
              + 4 * B * Lq * wl.H + 4 * B * Lq * Lk,
              "macs": pairs * wl.H * (2 * wl.d_qk + wl.d_v)}
        kl = {"bytes": 8 * pairs, "macs": 0.0}
        return {"indexer": ix, "dense_mla": dm, "indexer_kl": kl}
    sel = np.minimum(k, t + 1).astype(np.float64)  # selected entries per query
    pairs = B * vis.sum()
    nsel = B * sel.sum()
    ix = {"bytes": B * Lk * wl.d_I + B * Lq * wl.H_I * (wl.d_I + 4) + B * Lq * Lk * 4,
          "macs": pairs * wl.H_I * wl.d_I}
    tk = {"bytes": 4 * pairs + 4 * B * Lq * k, "macs": 0.0}
    # unique latents: in prefill every visible row of kv is selected by some query
    uniq_rows = B * min(Lk, nsel / B) if Lq == 1 else B * Lk
    ml = {"bytes": 2 * B * Lq * wl.H * wl.d_qk + 4 * B * Lq * k + 2 * uniq_rows * wl.d_qk
          + 2 * B * Lq * wl.H * wl.d_v + 4 * B * Lq * wl.H,
          "macs": nsel * wl.H * (wl.d_qk + wl.d_v)}
    if wl.emit_p:  # the p sweep recomputes Q K^T; p is written, KL reads scores at idx and p
        ml["macs"] += nsel * wl.H * wl.d_qk
        ml["bytes"] += 4 * B * Lq * k
    kl = {"bytes": 4 * nsel + 8 * B * Lq * k, "macs": 0.0}
    return {"indexer": ix, "topk": tk, "sparse_mla": ml, "indexer_kl": kl}


def _code_only(text: str) -> str:
    """C/C++/CUDA source with comments removed and whitespace runs collapsed."""
    import re

    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def source_hash():
    """Hash of the code (comments and layout ignored) of the CUDA sources and the C header:
    DRAM traffic recorded under profiles/ is reported only while the kernels it was measured on
    are unchanged."""
    import hashlib

    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "sparse_attention_tcgen05_b200", "csrc")
    for name in sorted(os.listdir(csrc)) + ["../../include/dsa.h"]:
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            h.update(name.encode() + b"\0" + _code_only(f.read()).encode())
    return h.hexdigest()[:12]


def measured_traffic(workload, kernel):
    """DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) of `kernel` on
    `workload` from profiles/dram_traffic.md, or None if absent or taken on other sources."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.md")
    if not os.path.exists(path):
        return None
    want = source_hash()
    for line in open(path):
        cells = [c.strip() for c in line.strip().strip("|").split("|")]
        if len(cells) >= 5 and cells[0] == workload and cells[1] == kernel and cells[4] == want:
            try:
                return float(cells[3])
            except ValueError:
                return None
    return None


def tensor_peak(stage, peaks, sustained):
    """Dense tensor peak (TFLOP/s) of a stage's contraction: bf16 for attention, FP8 (the bf16
    measurement times the datasheet's FP8/bf16 ratio) for the indexer; None for the rest."""
    bf16 = peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"]
    if stage in ("indexer", "indexer_topk"):
        return FP8_OVER_BF16 * bf16
    if stage in ("sparse_mla", "dense_mla"):
        return bf16
    return None


def roofline_us(stage, work, peaks, sustained=False):
    """Lower-bound time: slower of tensor time and HBM time at the measured copy bandwidth."""
    hbm_us = work["bytes"] / (peaks["hbm_gbs"] * 1e9) * 1e6
    tflops = tensor_peak(stage, peaks, sustained)
    tc_us = 2 * work["macs"] / (tflops * 1e12) * 1e6 if tflops else 0.0
    return max(hbm_us, tc_us), ("tensor" if tc_us > hbm_us else "hbm")


# ---------------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_id: str):
        self.proc = None
        self.dev = device_id
        self.path = os.path.join("/tmp", f"dsa_clocks_{os.getpid()}_{time.monotonic_ns()}.csv")

    def __enter__(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.fh,
                stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 7:
                    continue
                try:
                    sm.append(float(parts[0]))
                    smax.append(float(parts[1]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[3:7]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
        try:
            os.remove(self.path)
        except OSError:
            pass
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


def pci_id(device) -> str:
    """nvidia-smi --id value of a torch device (its PCI bus id; CUDA ordinals may be remapped)."""
    p = torch.cuda.get_device_properties(device)
    try:
        return f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
    except AttributeError:
        return str(device.index or 0)


# ---------------------------------------------------------------------------------- sharding
@dataclasses.dataclass
class Shard:
    """This rank's part of a job: the local workload the kernels are called with, and where its
    inputs sit in the job's seeded streams (sequences `seqs` of the job's workload, query rows
    [r0, r1) of each, keys [0, local.Lk))."""
    job: dsa_inputs.Workload     # the whole job (N * B sequences under weak scaling)
    local: dsa_inputs.Workload   # what this rank's kernels see
    seqs: list
    r0: int
    r1: int

    def describe(self):
        return {"seqs": [self.seqs[0], self.seqs[-1] + 1] if self.seqs else [0, 0],
                "rows": [self.r0, self.r1], "Lk": self.local.Lk}

    def global_rows(self):
        """Flat query rows (b * Lq + i) of the job that this rank computes."""
        return [b * self.job.Lq + i for b in self.seqs for i in range(self.r0, self.r1)]

    def host_inputs(self):
        job, loc = self.job, self.local
        n = self.r1 - self.r0
        qI = np.concatenate([dsa_inputs.q_index(job, b * job.Lq + self.r0, n) for b in self.seqs])
        w = np.concatenate([dsa_inputs.w_index(job, b * job.Lq + self.r0, n) for b in self.seqs])
        q = np.concatenate([dsa_inputs.q_attn(job, b * job.Lq + self.r0, n) for b in self.seqs])
        kI = np.stack([dsa_inputs.k_index(job, b)[:loc.Lk] for b in self.seqs])
        kv = np.stack([dsa_inputs.kv_latent(job, b)[:loc.Lk] for b in self.seqs])
        return {"qI": qI.reshape(loc.B, loc.Lq, loc.H_I, loc.d_I), "kI": kI,
                "w": w.reshape(loc.B, loc.Lq, loc.H_I), "q": q.reshape(loc.B, loc.Lq, loc.H, loc.d_qk),
                "kv": kv}


def make_shard(wl, rank, world, scaling):
    if scaling == "weak":
        job = dataclasses.replace(wl, B=wl.B * world)
        s0, s1 = shard_rows(job.B, rank, world)
        return Shard(job, dataclasses.replace(wl, B=s1 - s0), list(range(s0, s1)), 0, wl.Lq)
    if wl.Lq == 1:  # decode: one query per sequence, split the sequences
        s0, s1 = shard_rows(wl.B, rank, world)
        if s1 <= s0:
            raise SystemExit(f"strong scaling: {world} ranks for {wl.B} decode rows")
        return Shard(wl, dataclasses.replace(wl, B=s1 - s0), list(range(s0, s1)), 0, 1)
    # causal prefill: every sequence's query rows [start, stop), balanced by causal work; the
    # rank sees keys [0, stop + Lk - Lq), so row i of the shard keeps its position t
    start, stop = shard_causal_rows(wl.Lq, wl.Lk, wl.k, rank, world, mla_weight=MLA_WEIGHT)
    if stop <= start:
        raise SystemExit(f"strong scaling: {world} ranks for {wl.Lq} query rows")
    local = dataclasses.replace(wl, Lq=stop - start, Lk=stop + (wl.Lk - wl.Lq))
    return Shard(wl, local, list(range(wl.B)), start, stop)


# ---------------------------------------------------------------------------------- GPU arm
class Step:
    """Device buffers and the calls of one step through the C ABI."""

    def __init__(self, shard, device, keep_host=True):
        import sparse_attention_tcgen05_b200 as dsa

        wl = shard.local
        self.dsa, self.wl, self.dev = dsa, wl, device
        B, Lq, Lk = wl.B, wl.Lq, wl.Lk
        x = shard.host_inputs()
        h = {"qI": torch.from_numpy(x["qI"]).view(torch.float8_e4m3fn),
             "kI": torch.from_numpy(x["kI"]).view(torch.float8_e4m3fn),
             "w": torch.from_numpy(x["w"]),
             "q": torch.from_numpy(x["q"].view(np.int16)).view(torch.bfloat16),
             "kv": torch.from_numpy(x["kv"].view(np.int16)).view(torch.bfloat16)}
        del x
        # pinned host copies of the inputs (for the end-to-end measurement)
        self.h = {k_: v.pin_memory() for k_, v in h.items()} if keep_host else None
        self.d = {k_: v.to(device) for k_, v in (self.h or h).items()}
        del h
        self.scores = torch.empty(B, Lq, Lk, dtype=torch.float32, device=device)
        self.idx = None if wl.dense else torch.empty(B, Lq, wl.k, dtype=torch.int32, device=device)
        self.out = torch.empty(B, Lq, wl.H, wl.d_v, dtype=torch.bfloat16, device=device)
        self.lse = torch.empty(B, Lq, wl.H, dtype=torch.float32, device=device)
        pk = Lk if wl.dense else wl.k  # the dense target covers every position
        self.p = torch.empty(B, Lq, pk, dtype=torch.float32, device=device) if wl.emit_p else None
        self.loss = torch.empty(1, dtype=torch.float32, device=device)
        nws = max(dsa.dsa_workspace_bytes(dsa.DSA_OP_SPARSE_MLA_FWD, B, Lq, Lk, wl.k, wl.H),
                  dsa.dsa_workspace_bytes(dsa.DSA_OP_DENSE_MLA_FWD, B, Lq, Lk, 0, wl.H) if wl.dense else 0,
                  dsa.dsa_workspace_bytes(dsa.DSA_OP_INDEXER_KL, B, Lq, Lk, wl.k, 0), 16)
        self.ws = torch.empty(nws, dtype=torch.uint8, device=device)
        if keep_host:
            self.out_h = torch.empty(self.out.shape, dtype=torch.bfloat16).pin_memory()
            self.loss_h = torch.empty(1, dtype=torch.float32).pin_memory()
        self.reduce_loss = wl.emit_p and torch.distributed.is_initialized() and \
            torch.distributed.get_world_size() > 1
        # the split-KV combine is a separate launch only with more than two splits (two splits
        # combine inside the attention kernel)
        self.launches_per_step = (2 if wl.dense else 3) + (2 if wl.emit_p else 0) + \
            (1 if self._mla_splits() > 2 else 0)

    def _mla_splits(self):
        wl = self.wl
        if wl.emit_p or wl.dense:
            return 1
        ws = self.dsa.dsa_workspace_bytes(self.dsa.DSA_OP_SPARSE_MLA_FWD, wl.B, wl.Lq, wl.Lk, wl.k, wl.H)
        per_split = wl.rows * wl.H * (wl.d_v + 1) * 4  # partial O + lse of one split
        return max(1, ws // per_split) if ws else 1

    def run(self, ev=None):
        dsa, d, wl = self.dsa, self.d, self.wl
        if ev:
            ev[0].record()
        dsa.dsa_indexer(d["qI"], d["kI"], d["w"], self.scores)
        if ev:
            ev[1].record()
        if wl.dense:  # the dense warm-up step: no selection
            if ev:
                ev[2].record()
            dsa.dsa_dense_mla_fwd(d["q"], d["kv"], wl.scale, self.out, self.lse, self.p, self.ws)
            if ev:
                ev[3].record()
            dsa.dsa_indexer_kl_dense(self.scores, self.p, self.loss, None, self.ws)
            if self.reduce_loss:
                sum_over_ranks(self.loss)
            if ev:
                ev[4].record()
            return
        dsa.dsa_topk(self.scores, self.idx)
        if ev:
            ev[2].record()
        dsa.dsa_sparse_mla_fwd(d["q"], d["kv"], self.idx, wl.scale, self.out, self.lse, self.p, self.ws)
        if ev:
            ev[3].record()
        if wl.emit_p:
            dsa.dsa_indexer_kl(self.scores, self.idx, self.p, self.loss, None, self.ws)
            if self.reduce_loss:
                sum_over_ranks(self.loss)  # the sharded loss: one all-reduce of 4 bytes
        if ev:
            ev[4].record()

    def run_e2e(self):
        """Host buffers in, result out: H2D copies of this step's inputs, the path, D2H read."""
        for k_, v in self.h.items():
            self.d[k_].copy_(v, non_blocking=True)
        self.run()
        if self.wl.emit_p:
            self.loss_h.copy_(self.loss, non_blocking=True)
        else:
            self.out_h.copy_(self.out, non_blocking=True)

    def h2d_bytes(self):
        return sum(v.numel() * v.element_size() for v in self.h.values())

    def d2h_bytes(self):
        return 4 if self.wl.emit_p else self.out.numel() * 2


def cpu_oracle_sample(wl, budget_s=12.0, max_rows=None):
    """Time the fp64 oracle (as it stands) on a bounded sample of query rows of the workload,
    rows spread over the host cores.  Returns (qtok/s, cores, sample description)."""
    from oracle import oracle as ref

    cores = os.cpu_count() or 1
    rng = np.random.default_rng(17)
    pool = rng.permutation(wl.rows)
    kI = dsa_inputs.k_index(wl)
    kv = dsa_inputs.kv_latent(wl)

    def run(rows):
        qI = np.stack([dsa_inputs.q_index(wl, r, 1)[0] for r in rows])
        w = np.stack([dsa_inputs.w_index(wl, r, 1)[0] for r in rows])
        q = np.stack([dsa_inputs.q_attn(wl, r, 1)[0] for r in rows])
        t0 = time.perf_counter()
        ref.path_rows(wl, rows, qI, kI, w, q, kv, rows_packed=True, nthreads=min(cores, len(rows)),
                      want_scores=False)
        return time.perf_counter() - t0

    # calibrate on one row per core, then size the sample to the budget
    probe = [int(x) for x in pool[:cores]]
    dt = run(probe)
    n = max(cores, int(budget_s / max(dt, 1e-3) * cores))
    if max_rows:
        n = min(n, max_rows)
    n = min(n, wl.rows)
    rows = [int(x) for x in pool[:n]]
    dt = run(rows)
    return len(rows) / dt, cores, f"{len(rows)} of {wl.rows} query rows (seeded uniform), {dt:.1f} s"


def measure(shard, device, steps, warmup, world, peaks, e2e=True):
    """Times `steps` steps of the shard (after `warmup`), each between one pair of CUDA events on
    the launching stream with an L2 flush before it; returns the per-workload record."""
    wl = shard.local
    step = Step(shard, device, keep_host=e2e)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    for _ in range(warmup):
        step.run()
    torch.cuda.synchronize()
    # Timed region: each step's launches go back to back between one pair of events (events
    # between the kernels would stop each launch from overlapping the previous kernel's tail).
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(pci_id(device)) as clk:
        for i in range(steps):
            flush.fill_(i & 0xFF)  # evict L2 between steps (outside the step's events)
            evs[i][0].record()
            step.run()
            evs[i][1].record()
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    step_ms = [a.elapsed_time(b) for a, b in evs]
    # Per-stage times (for the stage roofline fractions) from a separate pass of the same steps
    # with an event between every two launches.
    attn = "dense_mla" if wl.dense else "sparse_mla"
    stage_ms = {"indexer": [], "topk": [], attn: [], "indexer_kl": []}
    for i in range(steps):
        flush.fill_(i & 0xFF)
        e = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
        step.run(e)
        torch.cuda.synchronize()
        stage_ms["indexer"].append(e[0].elapsed_time(e[1]))
        stage_ms["topk"].append(e[1].elapsed_time(e[2]))
        stage_ms[attn].append(e[2].elapsed_time(e[3]))
        stage_ms["indexer_kl"].append(e[3].elapsed_time(e[4]))
    if wl.dense:
        del stage_ms["topk"]
    total_ms = max_over_ranks(sum(step_ms), device)  # the slowest rank's time
    ms_per_step = total_ms / steps
    rows_all = shard.job.rows if world > 1 else wl.rows  # query rows of all ranks
    qtok = rows_all / (ms_per_step / 1e3)

    rec_e2e = None
    if e2e:
        e2e_steps = max(2, min(steps, 5))
        step.run_e2e()
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(e2e_steps):
            step.run_e2e()
        e1.record()
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, device)
        rec_e2e = {"value": rows_all / (e2e_ms / 1e3), "unit": "query-tokens/s",
                   "h2d_bytes_per_step": step.h2d_bytes(), "d2h_bytes_per_step": step.d2h_bytes()}

    # contractions are held to the burst GEMM peak (the stricter denominator); the sustained,
    # power-capped one is used only when the clocks sampled during the steps show the power cap
    # holding the SM clock well below its maximum
    c = clk.summary()
    sustained = bool(c.get("sm_mhz") and c.get("sm_max_mhz") and "sw_power_cap" in c.get("reasons", [])
                     and c["sm_mhz"] < 0.9 * c["sm_max_mhz"])
    work = algorithmic(wl)
    stages = {}
    for name, ms in stage_ms.items():
        if name == "indexer_kl" and not wl.emit_p:
            continue
        med = statistics.median(ms)
        r_us, bound = roofline_us(name, work[name], peaks, sustained)
        stages[name] = {"ms": round(med, 4), "roofline_us": round(r_us, 2), "bound": bound,
                        "frac": round(r_us / (med * 1e3), 4),
                        "gbs": round(work[name]["bytes"] / (med * 1e-3) / 1e9, 1),
                        "tflops": round(2 * work[name]["macs"] / (med * 1e-3) / 1e12, 1)}
        tp = tensor_peak(name, peaks, sustained)
        if tp:
            stages[name]["tensor_peak_tflops"] = round(tp, 1)
    path_roof = sum(v["roofline_us"] for v in stages.values())
    dom = max(stages, key=lambda s: stages[s]["ms"])
    ds = stages[dom]
    if ds["bound"] == "hbm":
        roof = {"kernel": dom, "bound": "hbm", "achieved": ds["gbs"], "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": round(ds["gbs"] / peaks["hbm_gbs"], 4)}
        src = peaks["source"] + " copy bandwidth"
    else:
        peak_t = tensor_peak(dom, peaks, sustained)
        roof = {"kernel": dom, "bound": "tensor", "achieved": ds["tflops"], "peak": round(peak_t, 1),
                "unit": "TFLOP/s", "frac": round(ds["tflops"] / peak_t, 4)}
        src = f"{peaks['source']} bf16 GEMM, {'sustained' if sustained else 'burst'}" + \
            (" x2 for fp8 (datasheet ratio)" if dom == "indexer" else "")
    roof["traffic"] = measured_traffic(wl.name, dom) if world == 1 else None
    roof["peak_source"] = src
    return {"workload": wl.name, "rows": rows_all, "steps": steps, "warmup": warmup,
            "ms_per_step": ms_per_step, "value": qtok, "unit": "query-tokens/s",
            "path_roofline_us": round(path_roof, 2),
            "path_roofline_frac": round(path_roof / (ms_per_step * 1e3), 4),
            "stages": stages, "roofline": roof, "clocks": c, "e2e": rec_e2e,
            "gpu_launches": step.launches_per_step * steps}


def time_calls(fn, steps, warmup, flush):
    """Median device time (ms) of fn() over `steps` calls after `warmup`, L2 flushed before each,
    CUDA events on the launching stream; also the clocks sampled meanwhile."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    ts = []
    with ClockSampler(pci_id(flush.device)) as clk:
        for i in range(steps):
            flush.fill_(i & 0xFF)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
    return statistics.median(ts), clk.summary()


def variant_blocks(device, peaks, steps, warmup):
    """The NEXT rows, each timed on its own: the indexer-loss backward on the sparse-stage
    workload's inputs, HISA's decode selection and a paged decode with ragged context lengths."""
    import sparse_attention_tcgen05_b200 as dsa

    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    out = {}
    bf16 = peaks["bf16_tflops"]

    # ---- indexer-loss backward (dq, dw, dk) after one sparse-stage forward
    wl = dsa_inputs.WORKLOADS["indexer_kl_16k"]
    st = Step(make_shard(wl, 0, 1, "weak"), device, keep_host=False)
    st.run()
    rows, Lk, k = wl.rows, wl.Lk, wl.k
    dq = torch.empty(wl.B, wl.Lq, wl.H_I, wl.d_I, device=device)
    dwt = torch.empty(wl.B, wl.Lq, wl.H_I, device=device)
    dk = torch.empty(wl.B, Lk, wl.d_I, device=device)
    d = st.d
    fn = lambda: dsa.dsa_indexer_bwd(d["qI"], d["kI"], d["w"], st.scores, st.idx, st.p, dq, dwt, dk)
    ms, clk = time_calls(fn, steps, warmup, flush)
    nsel = float(np.minimum(k, np.arange(wl.Lq) + 1).sum()) * wl.B
    macs8 = nsel * wl.H_I * wl.d_I                 # a = q . k recomputed (FP8)
    macs16 = 4 * nsel * wl.H_I * wl.d_I            # dq and dk, each on two fp16 parts
    tc_us = (2 * macs8 / (FP8_OVER_BF16 * bf16 * 1e12) + 2 * macs16 / (bf16 * 1e12)) * 1e6
    byts = rows * wl.H_I * (wl.d_I + 4) + Lk * wl.d_I + rows * k * 12 + rows * wl.H_I * (wl.d_I + 1) * 4 + \
        Lk * wl.d_I * 4 * 2
    hbm_us = byts / (peaks["hbm_gbs"] * 1e9) * 1e6
    out["indexer_bwd_16k"] = {
        "what": "dsa_indexer_bwd on indexer_kl_16k's own scores, idx and p (dq, dw, dk)", "ms": round(ms, 4),
        "roofline_us": round(max(tc_us, hbm_us), 1), "bound": "tensor" if tc_us > hbm_us else "hbm",
        "frac": round(max(tc_us, hbm_us) / (ms * 1e3), 4),
        "tflops": round(2 * (macs8 + macs16) / (ms * 1e-3) / 1e12, 1), "clocks": clk}
    del st, dq, dwt, dk
    torch.cuda.empty_cache()

    # ---- HISA and paged decode on the 128K decode workload
    wl = dsa_inputs.WORKLOADS["decode_128k"]
    st = Step(make_shard(wl, 0, 1, "weak"), device, keep_host=False)
    d = st.d
    B, L, k = wl.B, wl.Lk, wl.k
    st.run()  # the DSA selection, for the recall of HISA's
    dsa_idx = st.idx.clone()

    # the fused indexer -> top-k call (the indexer counts the top-k's first radix digit in its
    # epilogue) against the two separate calls, each step followed by the sparse MLA
    ws_ix = torch.zeros(max(16, dsa.dsa_workspace_bytes(dsa.DSA_OP_INDEXER_TOPK, B, 1, L, k, 0)),
                        dtype=torch.uint8, device=device)

    def fused_step():
        dsa.dsa_indexer_topk(d["qI"], d["kI"], d["w"], st.scores, st.idx, ws_ix)
        dsa.dsa_sparse_mla_fwd(d["q"], d["kv"], st.idx, wl.scale, st.out, st.lse, None, st.ws)

    ms_f, clk = time_calls(fused_step, steps, warmup, flush)
    same = bool(torch.equal(st.idx, dsa_idx))
    ms_s, _ = time_calls(st.run, steps, warmup, flush)
    out["decode_128k_fused_topk"] = {
        "what": "decode step with the fused indexer -> top-k call vs the separate calls (same selection)",
        "fused_ms_per_step": round(ms_f, 4), "separate_ms_per_step": round(ms_s, 4),
        "same_selection": same, "clocks": clk}
    block, r = 64, 64
    sums = torch.empty(B, L // block, wl.d_I, device=device)
    dsa.dsa_hisa_block_sums(d["kI"], block, sums)  # cache summary: once, outside the timed steps
    hidx = torch.empty(B, 1, k, dtype=torch.int32, device=device)
    hws = torch.zeros(dsa.dsa_hisa_workspace_bytes(B, L, block, r, k), dtype=torch.uint8, device=device)

    def hisa_step():
        dsa.dsa_hisa_topk(d["qI"], d["kI"], d["w"], sums, block, r, hidx, None, hws)
        dsa.dsa_sparse_mla_fwd(d["q"], d["kv"], hidx, wl.scale, st.out, st.lse, None, st.ws)

    ms, clk = time_calls(hisa_step, steps, warmup, flush)
    ms_sel, _ = time_calls(lambda: dsa.dsa_hisa_topk(d["qI"], d["kI"], d["w"], sums, block, r, hidx, None, hws),
                           steps, warmup, flush)
    a, b = dsa_idx.view(B, k), hidx.view(B, k)
    recall = float(np.mean([np.intersect1d(a[i].cpu().numpy(), b[i].cpu().numpy()).size / k for i in range(B)]))
    out["decode_128k_hisa"] = {
        "what": f"HISA selection (blocks of {block}, r = {r}: {r * block} candidate keys) + sparse MLA, "
                "block sums computed once outside the steps", "ms_per_step": round(ms, 4),
        "selection_ms": round(ms_sel, 4), "value": B / (ms * 1e-3), "unit": "query-tokens/s",
        "recall_vs_dsa": round(recall, 4), "clocks": clk}

    # paged cache: pages of 64 keys in a shuffled pool, context lengths uniform in [L/2, L]
    P = 64
    g = torch.Generator().manual_seed(0xD5A0 + 77)
    table = torch.randperm(B * (L // P), generator=g).to(torch.int32).reshape(B, L // P).to(device)
    lens = torch.randint(L // 2, L + 1, (B,), generator=g, dtype=torch.int32).to(device)
    kp = d["kI"].reshape(B * L // P, P, wl.d_I)
    kvp = d["kv"].reshape(B * L // P, P, wl.d_qk)
    pws = torch.zeros(dsa.dsa_workspace_bytes(dsa.DSA_OP_INDEXER_TOPK, B, 1, L, k, 0), dtype=torch.uint8,
                      device=device)

    def paged_step():
        dsa.dsa_indexer_topk_paged(d["qI"], kp, d["w"], table, lens, st.scores, st.idx, pws)
        dsa.dsa_sparse_mla_fwd_paged(d["q"], kvp, st.idx, table, lens, L, wl.scale, st.out, st.lse, st.ws)

    ms, clk = time_calls(paged_step, steps, warmup, flush)
    tot = float(lens.sum().item())
    byts = tot * wl.d_I + B * k * wl.d_qk * 2 + B * wl.H * (wl.d_qk + wl.d_v) * 2
    out["decode_128k_paged"] = {
        "what": f"paged decode, pages of {P} keys in a shuffled pool, seq_lens uniform in [{L // 2}, {L}] "
                f"(mean {tot / B:.0f})", "ms_per_step": round(ms, 4), "value": B / (ms * 1e-3),
        "unit": "query-tokens/s", "hbm_roofline_us": round(byts / (peaks["hbm_gbs"] * 1e9) * 1e6, 1),
        "clocks": clk}
    del st, kp, kvp
    torch.cuda.empty_cache()

    # ---- masked MHA (MHA mode, per-head keys and values) on a 4K prefill's own top-k sets,
    # against the MQA-mode sparse kernel on the same sets
    wl = dsa_inputs.WORKLOADS["prefill_1x4k"]
    st = Step(make_shard(wl, 0, 1, "weak"), device, keep_host=False)
    st.run()
    L, H, k = wl.Lk, wl.H, wl.k
    gen = lambda tid, shape: torch.from_numpy(
        dsa_inputs.normal_bf16_bits(wl.seed, tid, int(np.prod(shape))).view(np.int16).reshape(shape)).view(
        torch.bfloat16).to(device)
    qm, km, vm = gen(11, (1, L, H, 192)), gen(12, (1, L, H, 192)), gen(13, (1, L, H, 128))
    om = torch.empty(1, L, H, 128, dtype=torch.bfloat16, device=device)
    lm = torch.empty(1, L, H, device=device)
    mws = torch.empty(dsa.dsa_workspace_bytes(dsa.DSA_OP_MASKED_MHA, 1, L, L, k, H), dtype=torch.uint8,
                      device=device)
    ms_mha, clk = time_calls(lambda: dsa.dsa_masked_mha_fwd(qm, km, vm, st.idx, 1 / np.sqrt(192.0), om, lm, mws),
                             steps, warmup, flush)
    d = st.d
    ms_mqa, _ = time_calls(lambda: dsa.dsa_sparse_mla_fwd(d["q"], d["kv"], st.idx, wl.scale, st.out, st.lse, None,
                                                          st.ws), steps, warmup, flush)
    pairs = L * (L + 1) / 2
    nsel = float(np.minimum(k, np.arange(L) + 1).sum())
    fl_mha = 2 * pairs * H * (192 + 128)   # every causal (t, s) of the tiles the kernel visits
    fl_mqa = 2 * nsel * H * (576 + 512)
    out["prefill_4k_masked_mha"] = {
        "what": "masked MHA (MHA mode: 192-d keys, 128-d values per head) vs the MQA-mode sparse kernel, "
                "prefill_1x4k's own top-k sets", "masked_mha_ms": round(ms_mha, 4), "mqa_sparse_ms": round(ms_mqa, 4),
        "masked_mha_tflops": round(fl_mha / (ms_mha * 1e-3) / 1e12, 1),
        "masked_mha_tensor_frac": round(fl_mha / (ms_mha * 1e-3) / 1e12 / bf16, 4),
        "mqa_sparse_tflops": round(fl_mqa / (ms_mqa * 1e-3) / 1e12, 1), "clocks": clk}
    assert dsa.dsa_last_device_status() == 0
    return out


def workload_config(wl, world=1, scaling="weak", shard=None):
    cfg = {"workload": wl.name, "B": wl.B, "Lq": wl.Lq, "Lk": wl.Lk, "H_I": wl.H_I,
           "d_I": wl.d_I, "k": wl.k, "H": wl.H, "d_qk": wl.d_qk, "d_v": wl.d_v,
           "emit_p_and_kl": wl.emit_p, "l2": "flushed (512 MiB write) between steps, outside the step events",
           "stage_times": "separate pass with events between launches"}
    if world > 1:
        cfg["parallelism"] = f"rows over {world} ranks ({scaling} scaling)"
        cfg["job_rows"] = shard.job.rows
    return cfg


def gpu_arm(args, rank, world, device):
    wl = dsa_inputs.WORKLOADS[args.workload]
    shard = make_shard(wl, rank, world, args.scaling)
    peaks = load_peaks()
    rec = measure(shard, device, args.steps, args.warmup, world, peaks, e2e=True)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, cores, sample = cpu_oracle_sample(wl)
        cpu = {"value": v, "unit": "query-tokens/s", "cores": cores, "kind": "oracle", "sample": sample}
    line = {
        "metric": METRIC, "value": rec["value"], "unit": "query-tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": rec["ms_per_step"],
        "higher_is_better": True, "scaling": args.scaling, "vs_baseline": None,
        "dtype": "fp8e4m3 indexer, bf16 attention, fp32 accumulate", "data": "synthetic (seeded)",
        "config": workload_config(wl, world, args.scaling, shard),
        "e2e": rec["e2e"],
        "gpu_launches": rec["gpu_launches"],
        "roofline": rec["roofline"],
        "stages": rec["stages"],
        "path_roofline_us": rec["path_roofline_us"],
        "path_roofline_frac": rec["path_roofline_frac"],
        "clocks": rec["clocks"],
        "cpu_baseline": cpu,
    }
    if world == 1 and not args.no_extra:
        # every other workload, timed the same way (fewer steps, no host round trip)
        extra = {}
        names = [DECODE_TARGET] + [n for n in ("decode_32k", "prefill_2x8k", "indexer_kl_16k", "dense_warmup_16k",
                                            "tiny_prefill") if n != args.workload]
        for name in names:
            if name == args.workload:
                continue
            w2 = dsa_inputs.WORKLOADS[name]
            torch.cuda.empty_cache()
            r = measure(make_shard(w2, 0, 1, "weak"), device, args.extra_steps, max(3, args.warmup // 2),
                        1, peaks, e2e=False)
            r.pop("e2e")
            r["config"] = workload_config(w2)
            extra[name] = r
        if DECODE_TARGET in extra:
            line[DECODE_TARGET] = extra.pop(DECODE_TARGET)
            line[DECODE_TARGET]["target"] = "path_roofline_frac >= 0.60"
        line["workloads"] = extra
        line["gpu_launches"] += sum(r["gpu_launches"] for r in extra.values()) + \
            line.get(DECODE_TARGET, {}).get("gpu_launches", 0)
        torch.cuda.empty_cache()
        line["variants"] = variant_blocks(device, peaks, args.extra_steps, 3)
    return line


def reference_arm(args, world):
    wl = dsa_inputs.WORKLOADS[args.workload]
    budget = max(2.0, min(60.0, 20.0 / max(1, args.steps + args.warmup)))
    vals = []
    for i in range(args.warmup + args.steps):
        v, cores, sample = cpu_oracle_sample(wl, budget_s=budget)
        if i >= args.warmup:
            vals.append(v)
    v = statistics.median(vals)
    # the oracle runs on the host cores of rank 0; n_gpus is the launch's, as on the other arm
    return {"metric": METRIC, "value": v, "unit": "query-tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * wl.rows / v, "higher_is_better": True,
            "scaling": args.scaling, "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
            "config": workload_config(wl), "impl": "reference",
            "cpu_baseline": {"value": v, "unit": "query-tokens/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": v, "unit": "query-tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ---------------------------------------------------------------------------------- peaks
def peaks_arm(device):
    """Dense GEMM peaks (FP8 e4m3 via torch._scaled_mm, bf16 via torch.matmul; 8192^3, best of 10)
    and read-only / copy HBM references (torch.sum over 1 GiB and 4 GiB, copy_ of 1 GiB; best of
    10), all timed with CUDA events, with the clocks sampled during the loops."""
    def best(fn, reps=10):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        return min(ts), statistics.median(ts)

    res = {"metric": "measured peaks", "device": torch.cuda.get_device_name(device)}
    with ClockSampler(pci_id(device)) as clk:
        n = 8192
        a = torch.randn(n, n, device=device).to(torch.float8_e4m3fn)
        bt = torch.randn(n, n, device=device).to(torch.float8_e4m3fn).t()  # column-major B
        one = torch.ones((), device=device)
        t, tm = best(lambda: torch._scaled_mm(a, bt, scale_a=one, scale_b=one, out_dtype=torch.bfloat16))
        res["fp8_e4m3_tflops"] = {"best": 2 * n ** 3 / (t * 1e-3) / 1e12, "median": 2 * n ** 3 / (tm * 1e-3) / 1e12}
        del a, bt
        a = torch.randn(n, n, device=device, dtype=torch.bfloat16)
        b = torch.randn(n, n, device=device, dtype=torch.bfloat16)
        t, tm = best(lambda: torch.matmul(a, b))
        res["bf16_tflops"] = {"best": 2 * n ** 3 / (t * 1e-3) / 1e12, "median": 2 * n ** 3 / (tm * 1e-3) / 1e12}
        del a, b
        for gib in (1, 4):
            x = torch.ones(gib << 28, device=device, dtype=torch.float32)
            t, tm = best(lambda: torch.sum(x))
            res[f"hbm_read_sum_{gib}gib_gbs"] = {"best": (gib << 30) / (t * 1e-3) / 1e9,
                                                 "median": (gib << 30) / (tm * 1e-3) / 1e9}
            del x
        x = torch.ones(1 << 28, device=device, dtype=torch.float32)
        y = torch.empty_like(x)
        t, tm = best(lambda: y.copy_(x))
        res["hbm_copy_1gib_gbs"] = {"best": 2 * (1 << 30) / (t * 1e-3) / 1e9,
                                    "median": 2 * (1 << 30) / (tm * 1e-3) / 1e9}
        torch.cuda.synchronize()
    res["clocks"] = clk.summary()
    return res


# ---------------------------------------------------------------------------------- launcher
def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def relaunch(args):
    """Re-run this script under torch.distributed.run with one rank per GPU."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={args.gpus}",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), os.path.abspath(__file__),
           *sys.argv[1:]]
    return subprocess.call(cmd)


def dry_run(args, rank, world):
    """The launch and the sharding without CUDA: every rank reports its shard over gloo."""
    import datetime

    if world > 1:
        torch.distributed.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    wl = dsa_inputs.WORKLOADS[args.workload]
    sh = make_shard(wl, rank, world, args.scaling)
    mine = {"rank": rank, **sh.describe(), "global_rows": [min(sh.global_rows()), max(sh.global_rows()) + 1],
            "n_rows": len(sh.global_rows())}
    allv = [None] * world
    if world > 1:
        torch.distributed.all_gather_object(allv, mine)
    else:
        allv = [mine]
    if rank == 0:
        print(json.dumps({"dry_run": True, "n_gpus": world, "scaling": args.scaling, "workload": wl.name,
                          "job_rows": sh.job.rows, "shards": allv}), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--extra-steps", type=int, default=8, help="timed steps of each non-headline workload")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(dsa_inputs.WORKLOADS))
    ap.add_argument("--impl", default="dsa", choices=["dsa", "reference"])
    ap.add_argument("--scaling", default="weak", choices=["weak", "strong"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="time the headline workload only")
    ap.add_argument("--peaks", action="store_true", help="measure GEMM and HBM peaks instead")
    ap.add_argument("--dry-run", action="store_true", help="launch and shard without CUDA")
    args = ap.parse_args()
    if args.warmup < 3 and not args.dry_run:
        ap.error("--warmup must be at least 3")
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        sys.exit(relaunch(args))
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world != args.gpus:
        sys.exit(f"--gpus {args.gpus} but WORLD_SIZE {world}")
    if args.dry_run:
        dry_run(args, rank, world)
        return
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(reference_arm(args, world)), flush=True)
        return
    local = int(os.environ.get("LOCAL_RANK", "0"))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if args.peaks:
        if rank == 0:
            print(json.dumps(peaks_arm(device)), flush=True)
        return
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=device)
    line = gpu_arm(args, rank, world, device)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
