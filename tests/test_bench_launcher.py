"""bench.py's multi-GPU launch and sharding, on CPU: `--gpus 2 --dry-run` starts two ranks under
torch.distributed.run (gloo), every rank reports its shard, and the shards are disjoint and cover
every query row of the job.  A rank's shard of a causal sequence, run through the oracle with the
shard's own (Lq, Lk) and sliced inputs, gives the same rows as the whole sequence."""
import importlib.util
import json
import os
import subprocess
import sys

import numpy as np
import pytest

import dsa_inputs
from oracle import oracle as ref

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    sys.modules.setdefault("bench", mod)  # dataclasses look their module up by name
    spec.loader.exec_module(sys.modules["bench"])
    return sys.modules["bench"]


def _dry_run(workload, scaling, gpus=2):
    env = dict(os.environ, OMP_NUM_THREADS="1")
    env.pop("WORLD_SIZE", None)
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", str(gpus), "--dry-run",
                          "--workload", workload, "--scaling", scaling], capture_output=True, text=True,
                         timeout=240, env=env, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, out.stdout
    return json.loads(lines[0])


@pytest.mark.parametrize("workload,scaling", [("long_prefill_32k", "strong"), ("decode_32k", "weak"),
                                              ("decode_128k", "strong"), ("indexer_kl_16k", "weak")])
def test_two_ranks_cover_the_job_once(workload, scaling):
    res = _dry_run(workload, scaling)
    assert res["n_gpus"] == 2 and len(res["shards"]) == 2
    wl = dsa_inputs.WORKLOADS[workload]
    job_rows = wl.rows * (2 if scaling == "weak" else 1)
    assert res["job_rows"] == job_rows
    spans = sorted(tuple(s["global_rows"]) for s in res["shards"])
    # contiguous flat-row spans here (one sequence per rank, or rows of one sequence)
    assert spans[0][0] == 0 and spans[-1][1] == job_rows and spans[0][1] == spans[1][0]
    assert sum(s["n_rows"] for s in res["shards"]) == job_rows


def test_strong_prefill_shards_are_balanced_by_causal_work():
    bench = _bench()
    wl = dsa_inputs.WORKLOADS["long_prefill_32k"]
    shards = [bench.make_shard(wl, r, 4, "strong") for r in range(4)]
    assert [s.r0 for s in shards] == sorted(s.r0 for s in shards)
    assert shards[0].r0 == 0 and shards[-1].r1 == wl.Lq
    for s in shards:
        assert s.local.Lq == s.r1 - s.r0 and s.local.Lk == s.r1  # keys [0, stop)
    # later rows see more keys, so the later shards hold fewer rows
    sizes = [s.r1 - s.r0 for s in shards]
    assert sizes == sorted(sizes, reverse=True)


def test_a_causal_shard_reproduces_the_whole_sequence_rows():
    bench = _bench()
    wl = dsa_inputs.custom("shard_tiny", 0xD5A0 + 21, 1, 96, 96, 4, 32, 8, 16, 8, 80, 64, emit_p=True)
    world = 3
    full_q = dsa_inputs.q_attn(wl)
    whole = ref.path_rows(wl, list(range(wl.rows)), dsa_inputs.q_index(wl), dsa_inputs.k_index(wl),
                          dsa_inputs.w_index(wl), full_q, dsa_inputs.kv_latent(wl), rows_packed=False)
    for r in range(world):
        sh = bench.make_shard(wl, r, world, "strong")
        x = sh.host_inputs()
        loc = sh.local
        part = ref.path_rows(loc, list(range(loc.rows)), x["qI"].reshape(loc.rows, loc.H_I, loc.d_I),
                             x["kI"], x["w"].reshape(loc.rows, loc.H_I), x["q"].reshape(loc.rows, loc.H, loc.d_qk),
                             x["kv"], rows_packed=False)
        rows = slice(sh.r0, sh.r1)
        np.testing.assert_array_equal(part["idx"], whole["idx"][rows])
        np.testing.assert_array_equal(part["scores"], whole["scores"][rows, :loc.Lk])
        np.testing.assert_allclose(part["out"], whole["out"][rows], rtol=0, atol=0)
        np.testing.assert_allclose(part["kl"], whole["kl"][rows], rtol=0, atol=0)


def test_algorithmic_work_and_roofline_by_hand():
    # the per-stage byte and MAC counts the roofline fractions divide by, recomputed by hand for
    # the 128K decode rows and a causal prefill, and the bound each stage takes
    bench = _bench()
    wl = dsa_inputs.WORKLOADS["decode_128k"]
    w = bench.algorithmic(wl)
    B, L, k = 32, 131072, 2048
    assert w["indexer"]["bytes"] == B * L * 128 + B * 64 * (128 + 4) + B * L * 4
    assert w["indexer"]["macs"] == B * L * 64 * 128
    assert w["topk"]["bytes"] == 4 * B * L + 4 * B * k
    assert w["sparse_mla"]["macs"] == B * k * 128 * (576 + 512)
    # q + idx + the selected latents (k distinct rows per sequence) + out + lse
    assert w["sparse_mla"]["bytes"] == 2 * B * 128 * 576 + 4 * B * k + 2 * B * k * 576 + 2 * B * 128 * 512 + 4 * B * 128
    peaks = {"hbm_gbs": 6550.1, "bf16_tflops": 1660.8, "bf16_tflops_sustained": 1384.5}
    us, bound = bench.roofline_us("indexer", w["indexer"], peaks)
    assert bound == "hbm" and abs(us - w["indexer"]["bytes"] / 6550.1e3) < 1e-6
    us, bound = bench.roofline_us("sparse_mla", w["sparse_mla"], peaks)
    tc = 2 * w["sparse_mla"]["macs"] / 1660.8e6
    assert bound == ("tensor" if tc > w["sparse_mla"]["bytes"] / 6550.1e3 else "hbm")
    # causal prefill: pairs and selected entries summed over t = 0 .. L-1
    wl = dsa_inputs.WORKLOADS["prefill_2x8k"]
    w = bench.algorithmic(wl)
    L = 8192
    pairs = 2 * L * (L + 1) // 2
    nsel = 2 * sum(min(k, t + 1) for t in range(L))
    assert w["indexer"]["macs"] == pairs * 64 * 128
    assert w["sparse_mla"]["macs"] == nsel * 128 * 1088
    us, bound = bench.roofline_us("sparse_mla", w["sparse_mla"], peaks)
    assert bound == "tensor" and abs(us - 2 * nsel * 128 * 1088 / 1660.8e6) < 1e-6
    us, bound = bench.roofline_us("indexer", w["indexer"], peaks)  # FP8 at twice the bf16 figure
    assert bound == "tensor" and abs(us - 2 * pairs * 64 * 128 / (2 * 1660.8e6)) < 1e-6
