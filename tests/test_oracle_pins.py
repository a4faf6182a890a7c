"""Pins of the fp64 oracle against what the paper and mathematics fix.

Each test ties the oracle to something other than itself:
  * hand-derived worked examples (tests/golden/worked_examples.json),
  * library routines the method reduces to in special cases (torch's
    scaled_dot_product_attention for full / chunk-0 softmax, torch's elu for
    the feature map),
  * closed forms (linear attention through its cached sums, §3.1),
  * an independent recurrent implementation and a pure-Python brute force,
  * invariants (constant V, convex hull, linearity in V, set algebra).
The last block plants mistakes in the oracle and checks a pin catches each.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle.rehyat_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def _qkv(B, H, N, d, seed, scale=0.5):
    return _rand((B, H, N, d), seed, scale), _rand((B, H, N, d), seed + 1, scale), \
        _rand((B, H, N, d), seed + 2, 1.0)


def _sdpa(q, k, v):
    """Library full softmax attention in fp64 (scale 1/sqrt(d))."""
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x))
    return torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v)).numpy()


# --------------------------------------------------------------------------- #
# feature map                                                                  #
# --------------------------------------------------------------------------- #
def test_psi_closed_values():
    x = np.array([0.0, 1.0, 2.5, -1.0, -3.0, 1e-300, -1e-300])
    want = np.array([1.0, 2.0, 3.5, math.exp(-1.0), math.exp(-3.0), 1.0, 1.0])
    np.testing.assert_allclose(orc.psi(x), want, rtol=1e-15, atol=0)


def test_psi_is_one_plus_torch_elu():
    x = _rand((4096,), 3, 3.0)
    ref = 1.0 + torch.nn.functional.elu(torch.from_numpy(x)).numpy()
    np.testing.assert_allclose(orc.psi(x), ref, rtol=1e-15, atol=1e-15)


def test_phi_layout_and_nonnegative():
    x = _rand((7, 5), 4, 4.0)
    f = orc.phi(x)
    assert f.shape == (7, 10)
    ref = 1.0 + torch.nn.functional.elu(torch.from_numpy(x)).numpy()
    np.testing.assert_allclose(f[:, :5], ref, rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(f[:, 5:], ref ** 2, rtol=1e-14, atol=1e-15)
    assert (f > 0).all()


# --------------------------------------------------------------------------- #
# worked examples                                                              #
# --------------------------------------------------------------------------- #
def _golden_cases():
    with open(GOLDEN) as fh:
        return json.load(fh)["cases"]


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c["name"])
def test_golden_worked_examples(case):
    F, HW, Tc, To, d = case["F"], case["HW"], case["T_c"], case["T_o"], case["d"]
    q = np.array(case["q"], dtype=np.float64)[None, None]
    k = np.array(case["k"], dtype=np.float64)[None, None]
    v = np.array(case["v"], dtype=np.float64)[None, None]
    for mode, rows in case["expected"].items():
        want = np.array([[float(Fraction(x)) for x in r] for r in rows])
        got = orc.oracle_forward(q, k, v, F, HW, Tc, To, mode=mode)[0, 0]
        np.testing.assert_allclose(got, want, rtol=1e-13, atol=1e-13, err_msg=mode)
        bf = np.array(orc.oracle_bruteforce(q, k, v, F, HW, Tc, To, mode=mode))[0, 0]
        np.testing.assert_allclose(bf, want, rtol=1e-13, atol=1e-13, err_msg=mode)
        if mode == "causal":
            rec = orc.oracle_recurrent(q, k, v, F, HW, Tc, To)[0, 0]
            np.testing.assert_allclose(rec, want, rtol=1e-13, atol=1e-13)


# --------------------------------------------------------------------------- #
# reductions to library routines / closed forms                               #
# --------------------------------------------------------------------------- #
@pytest.mark.parametrize("mode", ["causal", "bidirectional"])
@pytest.mark.parametrize("F,HW,Tc,To", [(4, 8, 4, 1), (3, 16, 5, 0), (2, 5, 7, 3)])
def test_one_chunk_is_full_softmax(mode, F, HW, Tc, To):
    """P1: T_c >= F -> one chunk whose softmax set is every token."""
    q, k, v = _qkv(2, 2, F * HW, 16, 11)
    got = orc.oracle_forward(q, k, v, F, HW, Tc, To, mode=mode)
    np.testing.assert_allclose(got, _sdpa(q, k, v), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("F,HW,Tc,To", [(4, 6, 1, 0), (5, 4, 2, 1), (6, 3, 3, 2)])
def test_linear_only_is_cached_linear_attention(F, HW, Tc, To):
    """P2: with T^S empty the hybrid is §3.1 linear attention, evaluated here
    through its query-independent sums phi(K)^T V and sum phi(K)."""
    q, k, v = _qkv(1, 3, F * HW, 8, 21)
    got = orc.oracle_forward(q, k, v, F, HW, Tc, To, mode="linear_only")
    pq = 1.0 + torch.nn.functional.elu(torch.from_numpy(q)).numpy()
    pk = 1.0 + torch.nn.functional.elu(torch.from_numpy(k)).numpy()
    PQ = np.concatenate([pq, pq ** 2], -1)
    PK = np.concatenate([pk, pk ** 2], -1)
    kv = np.einsum("bhje,bhjc->bhec", PK, v)
    ks = PK.sum(axis=2)
    want = np.einsum("bhie,bhec->bhic", PQ, kv) / np.einsum("bhie,bhe->bhi", PQ, ks)[..., None]
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("F,HW,Tc,To", [(4, 8, 2, 1), (7, 5, 3, 1), (6, 4, 2, 3), (5, 3, 2, 0)])
def test_chunk0_rows_are_softmax_over_chunk0(F, HW, Tc, To):
    """P6 / reading R10: lo_0 = 0 so chunk 0 has no linear set."""
    q, k, v = _qkv(1, 2, F * HW, 16, 31)
    Np = min(Tc * HW, F * HW)
    got = orc.oracle_forward(q, k, v, F, HW, Tc, To, rows=np.arange(Np))
    want = _sdpa(q[:, :, :Np], k[:, :, :Np], v[:, :, :Np])
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


def test_softmax_window_of_later_chunk_matches_sdpa_when_linear_vanishes():
    """Chunk t >= 1 with the linear numerator/denominator removed is softmax
    over [lo_t, hi_t): checks the window bounds and the 1/sqrt(d) scale."""
    F, HW, Tc, To, d = 7, 6, 2, 1, 16
    q, k, v = _qkv(1, 1, F * HW, d, 41)
    aS, nS, _, _ = orc.oracle_parts(q, k, v, F, HW, Tc, To)
    for t in range(orc.n_chunks(F, Tc)):
        q0, q1, lo, hi = orc.chunk_geometry(t, F, HW, Tc, To)
        want = _sdpa(q[:, :, q0:q1], k[:, :, lo:hi], v[:, :, lo:hi])
        np.testing.assert_allclose(aS[:, :, q0:q1] / nS[:, :, q0:q1, None], want,
                                   rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------- #
# independent implementations                                                  #
# --------------------------------------------------------------------------- #
CFGS = [(4, 8, 2, 1), (7, 5, 3, 1), (6, 4, 2, 3), (5, 3, 2, 0), (3, 7, 1, 1), (5, 4, 5, 2),
        (8, 2, 3, 4), (1, 9, 2, 1)]


@pytest.mark.parametrize("F,HW,Tc,To", CFGS)
def test_recurrent_equals_parallel(F, HW, Tc, To):
    """P3: the §3.3 RNN form equals the explicit-mask parallel form."""
    q, k, v = _qkv(2, 2, F * HW, 8, 51)
    par = orc.oracle_forward(q, k, v, F, HW, Tc, To)
    rec = orc.oracle_recurrent(q, k, v, F, HW, Tc, To)
    np.testing.assert_allclose(rec, par, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("mode", ["causal", "bidirectional", "linear_only"])
@pytest.mark.parametrize("F,HW,Tc,To", [(4, 4, 2, 1), (5, 3, 2, 3), (3, 5, 1, 0)])
def test_bruteforce_equals_mask_oracle(mode, F, HW, Tc, To):
    """P4: inline set membership, scalar loops == explicit mask oracle."""
    q, k, v = _qkv(1, 2, F * HW, 4, 61)
    got = orc.oracle_forward(q, k, v, F, HW, Tc, To, mode=mode)
    bf = np.array(orc.oracle_bruteforce(q, k, v, F, HW, Tc, To, mode=mode))
    np.testing.assert_allclose(got, bf, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("F,HW,Tc,To", [(7, 5, 3, 1), (6, 4, 2, 3), (9, 2, 2, 0)])
def test_step_chain_equals_recurrent(F, HW, Tc, To):
    """The step call's framing (ctx/q/evict frames) reproduces the RNN form."""
    B, H, d = 1, 2, 8
    q, k, v = _qkv(B, H, F * HW, d, 71)
    want = orc.oracle_recurrent(q, k, v, F, HW, Tc, To)
    S = np.zeros((B, H, 2 * d, d))
    z = np.zeros((B, H, 2 * d))
    out = np.zeros_like(q)
    nc = orc.n_chunks(F, Tc)
    for t in range(nc):
        q0, q1, lo, hi = orc.chunk_geometry(t, F, HW, Tc, To)
        lo_next = orc.chunk_geometry(t + 1, F, HW, Tc, To)[2] if t + 1 < nc else hi
        evict = (min(lo_next, hi) - lo) // HW
        o, S, z = orc.oracle_step(q[:, :, q0:q1], k[:, :, lo:hi], v[:, :, lo:hi], S, z, HW, evict)
        out[:, :, q0:q1] = o
    np.testing.assert_allclose(out, want, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("F,HW,Tc,To", [(7, 5, 3, 1), (6, 4, 2, 3)])
def test_chunk_states_by_definition(F, HW, Tc, To):
    """S_t, z_t equal the explicit sums over the causal linear set (loops)."""
    q, k, v = _qkv(1, 1, F * HW, 3, 81)
    S, z = orc.oracle_chunk_states(k, v, F, HW, Tc, To)
    for t in range(orc.n_chunks(F, Tc)):
        lo = max(t * Tc * HW - To * HW, 0)
        Sw = np.zeros((6, 3))
        zw = np.zeros(6)
        for j in range(lo):
            f = [orc.psi(x) for x in k[0, 0, j]]
            f = f + [x * x for x in f]
            for e in range(6):
                zw[e] += f[e]
                for c in range(3):
                    Sw[e, c] += f[e] * v[0, 0, j, c]
        np.testing.assert_allclose(S[0, 0, t], Sw, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(z[0, 0, t], zw, rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------- #
# invariants                                                                   #
# --------------------------------------------------------------------------- #
@pytest.mark.parametrize("mode", ["causal", "bidirectional"])
def test_constant_v_and_convex_hull(mode):
    """P5: positive weights, jointly normalised -> y is a convex combination."""
    F, HW, Tc, To, d = 6, 5, 2, 1, 8
    q, k, v = _qkv(1, 2, F * HW, d, 91)
    c = np.linspace(-2.0, 3.0, d)
    got = orc.oracle_forward(q, k, np.broadcast_to(c, v.shape).copy(), F, HW, Tc, To, mode=mode)
    np.testing.assert_allclose(got, np.broadcast_to(c, got.shape), rtol=1e-13, atol=1e-13)
    y = orc.oracle_forward(q, k, v, F, HW, Tc, To, mode=mode)
    in_S, in_L = orc.hybrid_mask_rows(np.arange(F * HW), F, HW, Tc, To, mode)
    sel = in_S | in_L
    for b in range(1):
        for h in range(2):
            for i in range(F * HW):
                vv = v[b, h][sel[i]]
                assert (y[b, h, i] <= vv.max(0) + 1e-12).all()
                assert (y[b, h, i] >= vv.min(0) - 1e-12).all()


def test_linearity_in_v():
    """P8: y(aV1 + bV2) = a y(V1) + b y(V2) (the weights do not depend on V)."""
    F, HW, Tc, To, d = 5, 4, 2, 1, 8
    q, k, v1 = _qkv(1, 1, F * HW, d, 101)
    v2 = _rand(v1.shape, 102)
    f = lambda vv: orc.oracle_forward(q, k, vv, F, HW, Tc, To)
    np.testing.assert_allclose(f(2.5 * v1 - 0.75 * v2), 2.5 * f(v1) - 0.75 * f(v2),
                               rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("F,HW,Tc", [(6, 4, 2), (7, 3, 3), (5, 2, 1)])
def test_no_overlap_sets_match_paper_without_overlap(F, HW, Tc):
    """P7: with T_o = 0 the §3.2 overlap sets are the §3.2 sets without
    overlap: T^S_t = {tN' <= j < (t+1)N'}, T^L_t = T - T^S_t (built here
    directly), and causal T^L_t = {j < tN'}."""
    N, Np = F * HW, Tc * HW
    S, L = orc.hybrid_mask_rows(np.arange(N), F, HW, Tc, 0, "bidirectional")
    Sc, Lc = orc.hybrid_mask_rows(np.arange(N), F, HW, Tc, 0, "causal")
    for i in range(N):
        t = i // Np
        want_S = np.array([t * Np <= j < (t + 1) * Np for j in range(N)])
        np.testing.assert_array_equal(S[i], want_S)
        np.testing.assert_array_equal(L[i], ~want_S)
        np.testing.assert_array_equal(Sc[i], want_S)
        np.testing.assert_array_equal(Lc[i], np.arange(N) < t * Np)


def test_mask_partitions_tokens():
    """Causal: T^S and T^L are disjoint and together are [0, hi_t);
    bidirectional: they partition T; every query is in its own softmax set."""
    F, HW, Tc, To = 7, 3, 2, 3
    N = F * HW
    S, L = orc.hybrid_mask_rows(np.arange(N), F, HW, Tc, To, "causal")
    assert not (S & L).any()
    for i in range(N):
        assert S[i, i]
        hi = min((i // (Tc * HW) + 1) * Tc * HW, N)
        np.testing.assert_array_equal((S | L)[i], np.arange(N) < hi)
    S, L = orc.hybrid_mask_rows(np.arange(N), F, HW, Tc, To, "bidirectional")
    assert (S ^ L).all()


# --------------------------------------------------------------------------- #
# planted mistakes: each must be caught by at least one pin above              #
# --------------------------------------------------------------------------- #
def _pins_hold():
    """Run a compact subset of the pins; False if any disagrees."""
    try:
        for case in _golden_cases():
            test_golden_worked_examples(case)
        test_one_chunk_is_full_softmax("causal", 4, 8, 4, 1)
        test_recurrent_equals_parallel(7, 5, 3, 1)
        test_bruteforce_equals_mask_oracle("causal", 5, 3, 2, 3)
        test_linear_only_is_cached_linear_attention(5, 4, 2, 1)
        test_chunk0_rows_are_softmax_over_chunk0(7, 5, 3, 1)
    except AssertionError:
        return False
    return True


def test_unmodified_oracle_passes_compact_pins():
    assert _pins_hold()


def _mutant_mask(kind):
    orig = orc.hybrid_mask_rows

    def m(rows, F, HW, T_c, T_o, mode="causal"):
        if kind == "overlap_sign":
            return orig(rows, F, HW, T_c, -T_o, mode)
        if kind == "no_overlap":
            return orig(rows, F, HW, T_c, 0, mode)
        if kind == "drop_linear":
            S, L = orig(rows, F, HW, T_c, T_o, mode)
            return S, np.zeros_like(L)
        raise ValueError(kind)
    return m


MUTANTS = {
    "psi_without_one": ("psi", lambda x: np.where(np.asarray(x) > 0, x, np.exp(np.minimum(x, 0)) - 1.0)),
    "phi_drops_square": ("phi", lambda x: np.concatenate([orc.psi(x), orc.psi(x)], -1)),
    "phi_square_on_x": ("phi", lambda x: np.concatenate([orc.psi(x), np.asarray(x) ** 2], -1)),
    "overlap_sign": ("hybrid_mask_rows", _mutant_mask("overlap_sign")),
    "overlap_ignored": ("hybrid_mask_rows", _mutant_mask("no_overlap")),
    "linear_set_dropped": ("hybrid_mask_rows", _mutant_mask("drop_linear")),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(orc, attr, fn)
    assert not _pins_hold(), f"planted mistake {name} went unnoticed"


def test_planted_scale_mistake_is_caught(monkeypatch):
    """Queries pre-scaled by 1/sqrt(d) in the parallel oracle (scores then
    carry 1/d and phi sees scaled queries)."""
    orig_parts = orc.oracle_parts

    def parts(q, k, v, F, HW, T_c, T_o, mode="causal", rows=None, block=512, phi_q=None, phi_k=None):
        d = np.asarray(q).shape[-1]
        s = 1.0 / math.sqrt(d)
        return orig_parts(np.asarray(q) * s, k, v, F, HW, T_c, T_o, mode, rows, block, phi_q, phi_k)
    monkeypatch.setattr(orc, "oracle_parts", parts)
    assert not _pins_hold()


def test_planted_transposed_kv_is_caught(monkeypatch):
    """Keys and values swapped inside the parallel oracle."""
    orig_parts = orc.oracle_parts

    def parts(q, k, v, F, HW, T_c, T_o, mode="causal", rows=None, block=512, phi_q=None, phi_k=None):
        return orig_parts(q, v, k, F, HW, T_c, T_o, mode, rows, block, phi_q, phi_k)
    monkeypatch.setattr(orc, "oracle_parts", parts)
    assert not _pins_hold()


# --------------------------------------------------------------------------- #
# learned feature map: two-layer MLP with degree-2 polynomial features         #
# --------------------------------------------------------------------------- #
def _mlp_weights(H, d, seed, scale=1.0):
    """Random (non-symmetric) per-head weights, W1 [H,2d,d], W2 [H,2d,2d]."""
    g = np.random.default_rng(seed)
    return (g.standard_normal((H, 2 * d, d)) * scale / math.sqrt(d), g.standard_normal((H, 2 * d)) * 0.3,
            g.standard_normal((H, 2 * d, 2 * d)) * scale / math.sqrt(2 * d), g.standard_normal((H, 2 * d)) * 0.3)


def _maps(Wq, Wk):
    fq = lambda x, h: orc.phi_mlp(x, Wq[0][h], Wq[1][h], Wq[2][h], Wq[3][h])
    fk = lambda x, h: orc.phi_mlp(x, Wk[0][h], Wk[1][h], Wk[2][h], Wk[3][h])
    return fq, fk


@pytest.mark.parametrize("d", [3, 8])
def test_phi_mlp_matches_torch_modules(d):
    """phi_mlp == torch.nn.Linear -> ReLU -> Linear, then 1 + torch elu on
    each output half and the square of the second (P = 2 of the §3.2
    feature-map equation), in fp64 with the same weights."""
    W1, b1, W2, b2 = (w[0] for w in _mlp_weights(1, d, 5 + d))
    x = _rand((13, d), 7 + d, 2.0)
    l1 = torch.nn.Linear(d, 2 * d).double()
    l2 = torch.nn.Linear(2 * d, 2 * d).double()
    with torch.no_grad():
        l1.weight.copy_(torch.from_numpy(W1))
        l1.bias.copy_(torch.from_numpy(b1))
        l2.weight.copy_(torch.from_numpy(W2))
        l2.bias.copy_(torch.from_numpy(b2))
        u = l2(torch.relu(l1(torch.from_numpy(x))))
        p1 = 1.0 + torch.nn.functional.elu(u[:, :d])
        p2 = 1.0 + torch.nn.functional.elu(u[:, d:])
        want = torch.cat([p1, p2 ** 2], dim=1).numpy()
    got = orc.phi_mlp(x, W1, b1, W2, b2)
    np.testing.assert_allclose(got, want, rtol=1e-14, atol=1e-14)
    assert (got >= 0).all()


def test_phi_mlp_identity_weights_reduce_to_fixed_phi():
    """With W1 = [I; -I], W2 rows [I, -I] and zero biases the MLP outputs
    u = x, so the learned map is exactly the fixed phi, and the forward with
    those maps is the fixed-phi forward."""
    d = 6
    x = _rand((40, d), 11, 3.0)
    np.testing.assert_array_equal(orc.phi_mlp(x, *orc.mlp_identity_weights(d)), orc.phi(x))
    q, k, v = _qkv(1, 2, 20, d, 13)
    f = lambda x, h: orc.phi_mlp(x, *orc.mlp_identity_weights(d))
    np.testing.assert_allclose(orc.oracle_forward(q, k, v, 5, 4, 2, 1, phi_q=f, phi_k=f),
                               orc.oracle_forward(q, k, v, 5, 4, 2, 1), rtol=1e-13, atol=1e-14)


@pytest.mark.parametrize("F,HW,Tc,To", [(5, 4, 2, 1), (6, 3, 1, 2)])
def test_constant_features_closed_form(F, HW, Tc, To):
    """W2 = 0: every token gets the same features c = [psi(b2_1), psi(b2_2)^2].
    Linear-only attention is then the plain mean of V; in the causal sets every
    linear key weighs |c|^2, so y_i = (sum_S e^s v + |c|^2 sum_L v) /
    (sum_S e^s + |c|^2 |L|) with the sets counted from the §3.3 definitions."""
    d, N = 4, F * HW
    q, k, v = _qkv(1, 1, N, d, 17)
    W1, b1, W2, b2 = (w[0] for w in _mlp_weights(1, d, 19))
    W2 = np.zeros_like(W2)
    f = lambda x, h: orc.phi_mlp(x, W1, b1, W2, b2)
    lin = orc.oracle_forward(q, k, v, F, HW, Tc, To, mode="linear_only", phi_q=f, phi_k=f)
    np.testing.assert_allclose(lin[0, 0], np.broadcast_to(v[0, 0].mean(axis=0), (N, d)), rtol=1e-12)
    c = np.concatenate([orc.psi(b2[:d]), orc.psi(b2[d:]) ** 2])
    w = float(c @ c)
    got = orc.oracle_forward(q, k, v, F, HW, Tc, To, phi_q=f, phi_k=f)[0, 0]
    Np = Tc * HW
    for i in range(N):
        t = i // Np
        lo, hi = max(t * Np - To * HW, 0), min((t + 1) * Np, N)
        e = np.exp(k[0, 0, lo:hi] @ q[0, 0, i] / math.sqrt(d))
        num = e @ v[0, 0, lo:hi] + w * v[0, 0, :lo].sum(axis=0)
        den = e.sum() + w * lo
        np.testing.assert_allclose(got[i], num / den, rtol=1e-12)


@pytest.mark.parametrize("F,HW,Tc,To", [(7, 5, 3, 1), (6, 4, 2, 3), (5, 3, 1, 0)])
def test_mlp_recurrent_equals_parallel(F, HW, Tc, To):
    """§3.3 RNN form == explicit-mask parallel form with separate learned
    phi_q and phi_k per head."""
    d, H = 5, 2
    q, k, v = _qkv(1, H, F * HW, d, 23)
    fq, fk = _maps(_mlp_weights(H, d, 29), _mlp_weights(H, d, 31))
    par = orc.oracle_forward(q, k, v, F, HW, Tc, To, phi_q=fq, phi_k=fk)
    rec = orc.oracle_recurrent(q, k, v, F, HW, Tc, To, phi_q=fq, phi_k=fk)
    np.testing.assert_allclose(rec, par, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("mode", ["causal", "bidirectional", "linear_only"])
def test_mlp_bruteforce_equals_mask_oracle(mode):
    """Scalar loops with per-pair feature dot products == mask oracle, with
    phi_q != phi_k (a swap of the two maps changes the result)."""
    F, HW, Tc, To, d, H = 4, 3, 2, 1, 3, 2
    q, k, v = _qkv(1, H, F * HW, d, 37)
    fq, fk = _maps(_mlp_weights(H, d, 41), _mlp_weights(H, d, 43))
    got = orc.oracle_forward(q, k, v, F, HW, Tc, To, mode=mode, phi_q=fq, phi_k=fk)
    bf = np.array(orc.oracle_bruteforce(q, k, v, F, HW, Tc, To, mode=mode, phi_q=fq, phi_k=fk))
    np.testing.assert_allclose(got, bf, rtol=1e-12, atol=1e-13)
    swapped = orc.oracle_forward(q, k, v, F, HW, Tc, To, mode=mode, phi_q=fk, phi_k=fq)
    assert np.abs(swapped - bf).max() > 1e-6


def test_precomputed_feature_arrays_equal_maps():
    """Feature arrays [B,H,N,D'] stand in for the maps that produced them, in
    the parallel and the recurrent form."""
    F, HW, Tc, To, d, H = 5, 4, 2, 1, 4, 2
    q, k, v = _qkv(2, H, F * HW, d, 47)
    fq, fk = _maps(_mlp_weights(H, d, 53), _mlp_weights(H, d, 59))
    Pq = np.stack([np.stack([fq(q[b, h], h) for h in range(H)]) for b in range(2)])
    Pk = np.stack([np.stack([fk(k[b, h], h) for h in range(H)]) for b in range(2)])
    want = orc.oracle_forward(q, k, v, F, HW, Tc, To, phi_q=fq, phi_k=fk)
    np.testing.assert_allclose(orc.oracle_forward(q, k, v, F, HW, Tc, To, phi_q=Pq, phi_k=Pk, block=7), want,
                               rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(orc.oracle_recurrent(q, k, v, F, HW, Tc, To, phi_q=Pq, phi_k=Pk), want,
                               rtol=1e-12, atol=1e-13)


def _mlp_pins_hold():
    try:
        test_phi_mlp_matches_torch_modules(3)
        test_constant_features_closed_form(5, 4, 2, 1)
        test_mlp_bruteforce_equals_mask_oracle("causal")
    except AssertionError:
        return False
    return True


def test_unmodified_mlp_oracle_passes_pins():
    assert _mlp_pins_hold()


def _mlp_mutant(kind):
    orig = orc.phi_mlp

    def m(x, W1, b1, W2, b2):
        W1, W2 = np.asarray(W1), np.asarray(W2)
        if kind == "no_hidden_bias":
            return orig(x, W1, np.zeros_like(b1), W2, b2)
        if kind == "transposed_w2":
            return orig(x, W1, b1, W2.T, b2)
        if kind == "no_relu":
            x = np.asarray(x, dtype=np.float64)
            d = x.shape[-1]
            u = (x @ W1.T + b1) @ W2.T + b2
            return np.concatenate([orc.psi(u[..., :d]), orc.psi(u[..., d:]) ** 2], -1)
        if kind == "no_square":
            y = orig(x, W1, b1, W2, b2)
            d = y.shape[-1] // 2
            return np.concatenate([y[..., :d], np.sqrt(y[..., d:])], -1)
        raise ValueError(kind)
    return m


@pytest.mark.parametrize("kind", ["no_hidden_bias", "transposed_w2", "no_relu", "no_square"])
def test_planted_mlp_mistake_is_caught(kind, monkeypatch):
    monkeypatch.setattr(orc, "phi_mlp", _mlp_mutant(kind))
    assert not _mlp_pins_hold(), f"planted mistake {kind} went unnoticed"


def test_planted_swapped_maps_is_caught(monkeypatch):
    """phi_q and phi_k exchanged inside the parallel oracle."""
    orig_parts = orc.oracle_parts

    def parts(q, k, v, F, HW, T_c, T_o, mode="causal", rows=None, block=512, phi_q=None, phi_k=None):
        return orig_parts(q, k, v, F, HW, T_c, T_o, mode, rows, block, phi_k, phi_q)
    monkeypatch.setattr(orc, "oracle_parts", parts)
    assert not _mlp_pins_hold()
