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
