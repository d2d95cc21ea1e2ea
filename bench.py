"""Throughput of the DSA hot path on B200: query-tokens/s of one step = lightning indexer ->
top-k -> sparse MLA (and, for the sparse-stage workload, p emission + indexer KL) over one
batch of seeded synthetic inputs, plus each stage's roofline fraction.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl dsa|reference]

N > 1 runs under torchrun, one rank per GPU; every rank processes its own batch of the same
workload (weak scaling, no data-path collective) and the step time is the max over ranks.
`--impl reference` times the fp64 CPU oracle on a bounded sample of the same workload.
Prints ONE JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import dsa_inputs  # noqa: E402
from sparse_attention_tcgen05_b200.sharding import max_over_ranks  # noqa: E402

METRIC = "query-tokens/s (indexer+top-k+sparse MLA) at 1 B200; % of roofline per stage"
L2_FLUSH_BYTES = 512 << 20


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


def roofline_us(stage, work, peaks):
    """Lower-bound time: slower of tensor time (FP8 at 2x the measured bf16 dense peak for the
    indexer, bf16 for attention) and HBM time at the measured copy bandwidth."""
    hbm_us = work["bytes"] / (peaks["hbm_gbs"] * 1e9) * 1e6
    if stage == "indexer":
        tflops = 2 * peaks["bf16_tflops"]
    elif stage == "sparse_mla":
        tflops = peaks["bf16_tflops"]
    else:
        tflops = None
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
        self.path = os.path.join("/tmp", f"dsa_clocks_{os.getpid()}.csv")

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


# ---------------------------------------------------------------------------------- GPU arm
class Step:
    """Device buffers and the calls of one step through the C ABI."""

    def __init__(self, wl, device):
        import sparse_attention_tcgen05_b200 as dsa

        self.dsa, self.wl, self.dev = dsa, wl, device
        B, Lq, Lk = wl.B, wl.Lq, wl.Lk
        self.h = {  # pinned host copies of the inputs (for the end-to-end measurement)
            "qI": torch.from_numpy(dsa_inputs.q_index(wl).reshape(B, Lq, wl.H_I, wl.d_I)).view(
                torch.float8_e4m3fn).pin_memory(),
            "kI": torch.from_numpy(dsa_inputs.k_index(wl)).view(torch.float8_e4m3fn).pin_memory(),
            "w": torch.from_numpy(dsa_inputs.w_index(wl).reshape(B, Lq, wl.H_I)).pin_memory(),
            "q": torch.from_numpy(dsa_inputs.q_attn(wl).view(np.int16).reshape(B, Lq, wl.H, wl.d_qk)).view(
                torch.bfloat16).pin_memory(),
            "kv": torch.from_numpy(dsa_inputs.kv_latent(wl).view(np.int16)).view(torch.bfloat16).pin_memory(),
        }
        self.d = {k: v.to(device) for k, v in self.h.items()}
        self.scores = torch.empty(B, Lq, Lk, dtype=torch.float32, device=device)
        self.idx = torch.empty(B, Lq, wl.k, dtype=torch.int32, device=device)
        self.out = torch.empty(B, Lq, wl.H, wl.d_v, dtype=torch.bfloat16, device=device)
        self.lse = torch.empty(B, Lq, wl.H, dtype=torch.float32, device=device)
        self.p = torch.empty(B, Lq, wl.k, dtype=torch.float32, device=device) if wl.emit_p else None
        self.loss = torch.empty(1, dtype=torch.float32, device=device)
        nws = max(dsa.dsa_workspace_bytes(dsa.DSA_OP_SPARSE_MLA_FWD, B, Lq, Lk, wl.k, wl.H),
                  dsa.dsa_workspace_bytes(dsa.DSA_OP_INDEXER_KL, B, Lq, Lk, wl.k, 0), 16)
        self.ws = torch.empty(nws, dtype=torch.uint8, device=device)
        self.out_h = torch.empty(self.out.shape, dtype=torch.bfloat16).pin_memory()
        self.loss_h = torch.empty(1, dtype=torch.float32).pin_memory()
        # the split-KV combine is a separate launch only with more than two splits (two splits
        # combine inside the attention kernel)
        self.launches_per_step = 3 + (2 if wl.emit_p else 0) + (1 if self._mla_splits() > 2 else 0)

    def _mla_splits(self):
        wl = self.wl
        if wl.emit_p:
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
        dsa.dsa_topk(self.scores, self.idx)
        if ev:
            ev[2].record()
        dsa.dsa_sparse_mla_fwd(d["q"], d["kv"], self.idx, wl.scale, self.out, self.lse, self.p, self.ws)
        if ev:
            ev[3].record()
        if wl.emit_p:
            dsa.dsa_indexer_kl(self.scores, self.idx, self.p, self.loss, None, self.ws)
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
    rows_all = dsa_inputs.sample_rows(wl, 0) if wl.Lq > 1 else list(range(wl.rows))
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
    del rows_all
    return len(rows) / dt, cores, f"{len(rows)} of {wl.rows} query rows (seeded uniform), {dt:.1f} s"


def gpu_arm(args, rank, world, device):
    wl = dsa_inputs.WORKLOADS[args.workload]
    step = Step(wl, device)
    peaks = load_peaks()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    for _ in range(args.warmup):
        step.run()
    torch.cuda.synchronize()
    # Timed region: each step's launches go back to back between one pair of events (events
    # between the kernels would stop each launch from overlapping the previous kernel's tail).
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(pci_id(device)) as clk:
        for i in range(args.steps):
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
    stage_ms = {"indexer": [], "topk": [], "sparse_mla": [], "indexer_kl": []}
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        e = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
        step.run(e)
        torch.cuda.synchronize()
        stage_ms["indexer"].append(e[0].elapsed_time(e[1]))
        stage_ms["topk"].append(e[1].elapsed_time(e[2]))
        stage_ms["sparse_mla"].append(e[2].elapsed_time(e[3]))
        stage_ms["indexer_kl"].append(e[3].elapsed_time(e[4]))
    total_ms = max_over_ranks(sum(step_ms), device)  # the slowest rank's time
    ms_per_step = total_ms / args.steps
    qtok = wl.rows * world / (ms_per_step / 1e3)

    # end-to-end through host buffers
    e2e_steps = max(2, min(args.steps, 5))
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

    work = algorithmic(wl)
    stages = {}
    for name, ms in stage_ms.items():
        if name == "indexer_kl" and not wl.emit_p:
            continue
        med = statistics.median(ms)
        r_us, bound = roofline_us(name, work[name], peaks)
        stages[name] = {"ms": round(med, 4), "roofline_us": round(r_us, 2), "bound": bound,
                        "frac": round(r_us / (med * 1e3), 4),
                        "gbs": round(work[name]["bytes"] / (med * 1e-3) / 1e9, 1),
                        "tflops": round(2 * work[name]["macs"] / (med * 1e-3) / 1e12, 1)}
    path_roof = sum(v["roofline_us"] for v in stages.values())
    dom = max(stages, key=lambda s: stages[s]["ms"])
    ds = stages[dom]
    if ds["bound"] == "hbm":
        roof = {"kernel": dom, "bound": "hbm", "achieved": ds["gbs"], "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": round(ds["gbs"] / peaks["hbm_gbs"], 4)}
    else:
        peak_t = peaks["bf16_tflops"] * (2 if dom == "indexer" else 1)
        roof = {"kernel": dom, "bound": "tensor", "achieved": ds["tflops"], "peak": peak_t,
                "unit": "TFLOP/s", "frac": round(ds["tflops"] / peak_t, 4)}
    roof["traffic"] = measured_traffic(wl.name, dom)
    roof["peak_source"] = peaks["source"] + (" (fp8 = 2x measured bf16)" if roof["unit"] == "TFLOP/s" and dom == "indexer" else "")
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, cores, sample = cpu_oracle_sample(wl)
        cpu = {"value": v, "unit": "query-tokens/s", "cores": cores, "kind": "oracle", "sample": sample}
    line = {
        "metric": METRIC, "value": qtok, "unit": "query-tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "fp8e4m3 indexer, bf16 attention, fp32 accumulate", "data": "synthetic (seeded)",
        "config": workload_config(wl),
        "e2e": {"value": wl.rows * world / (e2e_ms / 1e3), "unit": "query-tokens/s",
                "h2d_bytes_per_step": step.h2d_bytes(), "d2h_bytes_per_step": step.d2h_bytes()},
        "gpu_launches": step.launches_per_step * args.steps,
        "roofline": roof,
        "stages": stages,
        "path_roofline_frac": round(path_roof / (ms_per_step * 1e3), 4),
        "clocks": clk.summary(),
        "cpu_baseline": cpu,
    }
    return line


def workload_config(wl):
    return {"workload": wl.name, "B": wl.B, "Lq": wl.Lq, "Lk": wl.Lk, "H_I": wl.H_I,
            "d_I": wl.d_I, "k": wl.k, "H": wl.H, "d_qk": wl.d_qk, "d_v": wl.d_v,
            "emit_p_and_kl": wl.emit_p, "l2": "flushed (512 MiB write) between steps, outside the step events",
            "stage_times": "separate pass with events between launches"}


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
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
            "config": workload_config(wl), "impl": "reference",
            "cpu_baseline": {"value": v, "unit": "query-tokens/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": v, "unit": "query-tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="decode_32k", choices=sorted(dsa_inputs.WORKLOADS))
    ap.add_argument("--impl", default="dsa", choices=["dsa", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(reference_arm(args, world)), flush=True)
        return
    local = int(os.environ.get("LOCAL_RANK", "0"))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
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
