"""The bench's algorithmic work (FLOPs and bytes behind every roofline
figure) counted independently: softmax pairs and linear-term rows from the
oracle's explicit hybrid mask, for both set modes, on small shapes."""
import numpy as np
import pytest

import bench
import oracle.rehyat_oracle as orc


CASES = [(4, 8, 2, 1), (7, 5, 3, 1), (6, 4, 2, 3), (5, 3, 2, 0), (21, 3, 3, 1), (9, 2, 4, 2), (3, 5, 5, 1)]


@pytest.mark.parametrize("F,S,Tc,To", CASES)
@pytest.mark.parametrize("sets", ["causal", "bidirectional"])
def test_pairs_and_linear_rows_match_the_mask(F, S, Tc, To, sets):
    c = dict(B=1, H=1, d=8, F=F, S_tok=S, T_c=Tc, T_o=To)
    w = bench.work(c, sets)
    N = F * S
    in_S, in_L = orc.hybrid_mask_rows(np.arange(N), F, S, Tc, To, sets)
    assert w["pairs_per_head"] == int(in_S.sum())
    d, D2 = 8, 16
    n_lin = int(in_L.any(axis=1).sum())
    # keys folded into linear states: every key some query reaches linearly
    folded = int(in_L.any(axis=0).sum()) if sets == "causal" else (N if -(-F // min(Tc, F)) > 1 else 0)
    assert w["attn_flops"] == 4 * d * int(in_S.sum()) + 2 * D2 * (d + 1) * n_lin
    assert w["state_flops"] == 2 * D2 * (d + 1) * folded
    assert w["tokens"] == N


def test_wan13b_work_figures():
    """The 1.3B-480p figures quoted with the bench line, by hand: 7 chunks of
    N' = 3 x 1560 = 4680 queries; chunk 0 sees its own 4680 keys, chunks 1-6
    also the 1560 keys of the overlap frame (6240); 12 heads, d = 128."""
    w = bench.work(dict(bench.CONFIGS["wan13b"]))
    pairs = 4680 * 4680 + 6 * 4680 * 6240
    assert w["pairs_per_head"] == pairs == 197_121_600
    n_lin = 6 * 4680                         # rows of chunks 1-6 have a linear term
    assert w["attn_flops"] == 12 * (4 * 128 * pairs + 2 * 256 * 129 * n_lin)
    # q, k, v, out once (bf16) + per chunk the bf16 hi and lo states and fp32 z
    assert w["attn_bytes"] == 12 * 32760 * 128 * 2 * 4 + 12 * 7 * 256 * (128 * 4 + 4)


# --------------------------------------------------------------------------- #
# the reference arm (the oracle on the host cores) keeps the line contract     #
# --------------------------------------------------------------------------- #
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench(*args, env=None):
    e = dict(os.environ)
    e.update(env or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True, text=True,
                          timeout=300, cwd=ROOT, env=e)


def test_reference_arm_prints_one_contract_line():
    r = _bench("--impl", "reference", "--steps", "1", "--warmup", "3", "--heads", "1", "--ref-budget", "1")
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    j = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in j, key
    assert j["impl"] == "reference" and j["value"] > 0 and j["steps"] == 1
    assert j["cpu_baseline"]["kind"] == "oracle" and j["cpu_baseline"]["value"] == j["value"]
    assert j["e2e"] == {"value": j["value"], "unit": j["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert j["config"]["H"] == 1 and "workload" in j["config"]


def test_reference_arm_other_ranks_exit_quietly():
    r = _bench("--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3", "--heads", "1",
               "--ref-budget", "1", env={"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r.returncode == 0, r.stderr
    assert not [l for l in r.stdout.splitlines() if l.startswith("{")]


def test_gpu_count_must_match_the_process_count():
    r = _bench("--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3", env={"WORLD_SIZE": "1"})
    assert r.returncode != 0 and "torch.distributed.run" in r.stderr
