"""GPU parity of the learned feature map (two-layer MLP, degree-2 features)
and of the hybrid forward that uses it, against the fp64 oracle.

The feature-map kernel is checked element by element against a bound derived
from its arithmetic (below); the forwards use the bf16 tolerances of the
other parity tests (relative L2 <= 1e-2, max |error| <= 3e-2 RMS).
"""
import numpy as np
import pytest
import torch

import oracle.rehyat_oracle as orc
from linear_attention_video_chunk_b200 import inputs
from linear_attention_video_chunk_b200 import rehyat as R
from test_gpu_parity import assert_bf16_close, few_rows, np64

pytestmark = pytest.mark.gpu

U_BF16 = 2.0 ** -8  # unit roundoff of bf16 (8-bit significand)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    R.lib()
    yield
    assert R.device_status() == R.OK, "a device-side wait timed out"


def _w64(w):
    return tuple(t.double().numpy() for t in w)


def _oracle_phi(x, w):
    """fp64 oracle features of x [B,H,N,d] with per-head weights -> [B,H,N,2d]."""
    W1, b1, W2, b2 = _w64(w)
    x = np.asarray(x.double().numpy() if isinstance(x, torch.Tensor) else x)
    return np.stack([np.stack([orc.phi_mlp(x[b, h], W1[h], b1[h], W2[h], b2[h]) for h in range(x.shape[1])])
                     for b in range(x.shape[0])])


def _bound(x, w, ref):
    """Elementwise error bound of the kernel's arithmetic.  The hidden units
    relu(W1 x + b1) are rounded to bf16 (relative error <= u = 2^-8) before
    the second GEMM, so |du_o| <= E_o = u * sum_j |W2[o,j]| |h_j|; 1 + elu is
    1-Lipschitz, and (psi^2)' = 2 psi; the output is rounded to bf16 once more
    (<= u |phi|).  fp32 accumulation and the fp32 exp add far less than the
    25% margin."""
    W1, b1, W2, b2 = _w64(w)
    x = x.double().numpy()
    B, H, N, d = x.shape
    tol = np.empty_like(ref)
    for b in range(B):
        for h in range(H):
            hid = np.maximum(x[b, h] @ W1[h].T + b1[h], 0.0)
            E = U_BF16 * (hid @ np.abs(W2[h]).T)
            psi2 = np.sqrt(ref[b, h, :, d:])
            tol[b, h, :, :d] = U_BF16 * ref[b, h, :, :d] + E[:, :d]
            tol[b, h, :, d:] = U_BF16 * ref[b, h, :, d:] + 2.0 * psi2 * E[:, d:] + E[:, d:] ** 2
    return 1.25 * tol + 1e-6


MLP_CASES = [
    # B, H, N, d, layout, kind, seed
    (2, 3, 300, 128, "bhnd", "near_identity", 1),   # ragged last tile (300 = 2 x 128 + 44)
    (1, 2, 1000, 128, "bnhd", "random", 2),         # [B, N, H, d] input
    (2, 2, 257, 64, "bhnd", "random", 3),           # d = 64, one-row last tile
    (1, 1, 128, 64, "bnhd", "near_identity", 4),    # exactly one tile
    (1, 1, 5, 128, "bhnd", "random", 5),            # fewer rows than a tile
    # 80 (map, b.h) pairs: one row group each, so every CTA walks all the
    # tiles of its head (the cross-tile overlap of the second U half and the
    # x reloads), the last one ragged
    (2, 40, 1000, 128, "bhnd", "random", 6),        # 8 tiles, 104-row last tile
    (1, 80, 700, 64, "bnhd", "near_identity", 7),   # d = 64: 6 tiles, 60-row last tile
]


@pytest.mark.parametrize("B,H,N,d,layout,kind,seed", MLP_CASES)
def test_phi_mlp_kernel_matches_oracle(B, H, N, d, layout, kind, seed):
    x = inputs.make_qkv(B, H, N, d, seed, rms_qk=True)[0]
    w = inputs.make_mlp_weights(H, d, seed, "q", kind)
    xin = x.transpose(1, 2).contiguous() if layout == "bnhd" else x
    y = R.phi_mlp(xin.cuda(), *(t.cuda() for t in w), layout=layout)
    torch.cuda.synchronize()
    ref = _oracle_phi(x, w)
    got = np64(y)
    assert (got >= 0).all()
    err = np.abs(got - ref)
    tol = _bound(x, w, ref)
    bad = err > tol
    assert not bad.any(), f"{bad.sum()} of {bad.size} features outside the bound; worst {(err / tol).max():.3f}"


def test_phi_mlp_identity_weights_give_fixed_phi():
    """W1 = [I; -I], W2 = [[I, -I]; [I, -I]], zero biases: every step is exact
    up to the final bf16 rounding, so the kernel returns the fixed phi of the
    bf16 inputs rounded to bf16 (the oracle's phi, cast by torch)."""
    B, H, N, d = 1, 2, 200, 128
    x = inputs.make_qkv(B, H, N, d, 9, rms_qk=True)[0]
    W1, b1, W2, b2 = orc.mlp_identity_weights(d)
    w = (torch.from_numpy(np.stack([W1] * H)).to(torch.bfloat16), torch.from_numpy(np.stack([b1] * H)).float(),
         torch.from_numpy(np.stack([W2] * H)).to(torch.bfloat16), torch.from_numpy(np.stack([b2] * H)).float())
    y = R.phi_mlp(x.cuda(), *(t.cuda() for t in w)).cpu()
    ref = torch.from_numpy(orc.phi(x.double().numpy())).to(torch.bfloat16)
    diff = (y.double() - ref.double()).abs()
    # psi is computed in fp32 (exp within a few ulp), then rounded: at most one bf16 ulp apart
    assert (diff <= 2.0 ** -7 * ref.double().abs() + 1e-30).all()


PHI_CASES = [
    # B, H, d, F, S_tok, Tc, To, sets, seed
    (1, 2, 128, 5, 200, 2, 1, "causal", 40),
    (1, 2, 64, 5, 200, 2, 1, "causal", 41),
    (2, 1, 128, 6, 70, 2, 3, "causal", 42),
    (1, 2, 128, 5, 200, 2, 1, "bidirectional", 43),
    (1, 1, 128, 3, 150, 4, 1, "causal", 44),        # one chunk: no linear set
]


def _bf16_features(x, w):
    return torch.from_numpy(_oracle_phi(x, w)).to(torch.bfloat16)


@pytest.mark.parametrize("B,H,d,F,S,Tc,To,sets,seed", PHI_CASES)
def test_forward_phi_matches_oracle(B, H, d, F, S, Tc, To, sets, seed):
    """Precomputed bf16 features (the oracle's MLP of the bf16 inputs, cast to
    bf16) fed to both sides."""
    q, k, v = inputs.make_qkv(B, H, F * S, d, seed, rms_qk=True)
    Pq = _bf16_features(q, inputs.make_mlp_weights(H, d, seed, "q"))
    Pk = _bf16_features(k, inputs.make_mlp_weights(H, d, seed, "k"))
    y = R.forward_phi(q.cuda(), k.cuda(), v.cuda(), Pq.cuda(), Pk.cuda(), F, S, Tc, To, sets=sets)
    mode = "causal" if sets == "causal" else "bidirectional"
    ref = orc.oracle_forward(q, k, v, F, S, Tc, To, mode=mode, phi_q=Pq.double().numpy(), phi_k=Pk.double().numpy())
    assert_bf16_close(np64(y), ref, f"forward_phi {sets}")


@pytest.mark.parametrize("layout", ["bhnd", "bnhd"])
def test_forward_mlp_is_phi_mlp_then_forward_phi(layout):
    """rehyat_forward_mlp == rehyat_phi_mlp of q and of k, then
    rehyat_forward_phi: bit for bit (the same kernels in the same order)."""
    B, H, d, F, S, Tc, To = 1, 2, 128, 6, 130, 3, 1
    q, k, v = (x.cuda() for x in inputs.make_qkv(B, H, F * S, d, 45, rms_qk=True))
    wq = tuple(t.cuda() for t in inputs.make_mlp_weights(H, d, 45, "q", "random"))
    wk = tuple(t.cuda() for t in inputs.make_mlp_weights(H, d, 45, "k", "random"))
    if layout == "bnhd":
        q, k, v = (x.transpose(1, 2).contiguous() for x in (q, k, v))
    y = R.forward_mlp(q, k, v, wq, wk, F, S, Tc, To, layout=layout)
    Pq = R.phi_mlp(q, *wq, layout=layout)
    Pk = R.phi_mlp(k, *wk, layout=layout)
    assert torch.equal(y, R.forward_phi(q, k, v, Pq, Pk, F, S, Tc, To, layout=layout))


MLP_FWD_CASES = [
    # B, H, d, F, S_tok, Tc, To, sets, kind, seed
    (1, 2, 128, 5, 200, 2, 1, "causal", "near_identity", 50),
    (1, 2, 64, 7, 90, 2, 3, "causal", "random", 51),
    (2, 1, 128, 6, 100, 3, 0, "bidirectional", "near_identity", 52),
]


@pytest.mark.parametrize("B,H,d,F,S,Tc,To,sets,kind,seed", MLP_FWD_CASES)
def test_forward_mlp_matches_oracle(B, H, d, F, S, Tc, To, sets, kind, seed):
    """End to end against the oracle's fp64 MLP features (no bf16 features on
    the oracle side)."""
    q, k, v = inputs.make_qkv(B, H, F * S, d, seed, rms_qk=True)
    wq = inputs.make_mlp_weights(H, d, seed, "q", kind)
    wk = inputs.make_mlp_weights(H, d, seed, "k", kind)
    y = R.forward_mlp(q.cuda(), k.cuda(), v.cuda(), tuple(t.cuda() for t in wq), tuple(t.cuda() for t in wk),
                      F, S, Tc, To, sets=sets)
    mode = "causal" if sets == "causal" else "bidirectional"
    ref = orc.oracle_forward(q, k, v, F, S, Tc, To, mode=mode, phi_q=_oracle_phi(q, wq), phi_k=_oracle_phi(k, wk))
    assert_bf16_close(np64(y), ref, f"forward_mlp {sets} {kind}")


def test_wan13b_480p_forward_mlp_sampled_rows():
    """The learned-map forward at the Wan2.1-1.3B 480p shape (B=1, H=12,
    d=128, 21 x 1560 tokens, T_c=3, T_o=1), sampled rows of every head."""
    B, H, d, F, S, Tc, To = 1, 12, 128, 21, 1560, 3, 1
    q, k, v = inputs.make_qkv(B, H, F * S, d, 1, rms_qk=True)
    wq = inputs.make_mlp_weights(H, d, 1, "q")
    wk = inputs.make_mlp_weights(H, d, 1, "k")
    y = R.forward_mlp(q.cuda(), k.cuda(), v.cuda(), tuple(t.cuda() for t in wq), tuple(t.cuda() for t in wk),
                      F, S, Tc, To).cpu()
    rows = few_rows(F, S, Tc)
    Pq = _oracle_phi(q, wq)[:, :, rows]
    Pk = _oracle_phi(k, wk)
    # the oracle indexes query features by row: give it a full-size array
    Pq_full = np.zeros(Pk.shape)
    Pq_full[:, :, rows] = Pq
    ref = orc.oracle_forward(q, k, v, F, S, Tc, To, rows=rows, phi_q=Pq_full, phi_k=Pk)
    assert_bf16_close(np64(y[:, :, rows]), ref, "wan13b forward_mlp")


def test_forward_mlp_identity_weights_close_to_fixed_phi():
    """Identity weights make the learned map the fixed phi; the only change is
    that phi(q) is rounded to bf16 before its exp(-M) scaling."""
    B, H, d, F, S, Tc, To = 1, 2, 128, 6, 130, 3, 1
    q, k, v = (x.cuda() for x in inputs.make_qkv(B, H, F * S, d, 46, rms_qk=True))
    W1, b1, W2, b2 = orc.mlp_identity_weights(d)
    w = (torch.from_numpy(np.stack([W1] * H)).to(torch.bfloat16).cuda(),
         torch.from_numpy(np.stack([b1] * H)).float().cuda(),
         torch.from_numpy(np.stack([W2] * H)).to(torch.bfloat16).cuda(),
         torch.from_numpy(np.stack([b2] * H)).float().cuda())
    y = R.forward_mlp(q, k, v, w, w, F, S, Tc, To)
    ref = R.forward(q, k, v, F, S, Tc, To)
    assert_bf16_close(np64(y), np64(ref), "identity weights vs fixed phi")


@pytest.mark.parametrize("F,S,Tc,To", [(8, 120, 3, 1), (7, 64, 2, 3), (6, 50, 1, 0)])
def test_step_phi_streamed_matches_oracle(F, S, Tc, To):
    """The recurrent form with learned features: chunk by chunk through
    rehyat_step_phi (features of each chunk's q and window k sliced from the
    video's), against the oracle (parallel == recurrent with the same bf16
    features), and against rehyat_forward_phi."""
    B, H, d = 1, 2, 128
    q, k, v = inputs.make_qkv(B, H, F * S, d, 71, rms_qk=True)
    Pq = _bf16_features(q, inputs.make_mlp_weights(H, d, 71, "q", "random"))
    Pk = _bf16_features(k, inputs.make_mlp_weights(H, d, 71, "k", "random"))
    qd, kd, vd, Pqd, Pkd = (x.cuda() for x in (q, k, v, Pq, Pk))
    Sst = torch.zeros(B, H, 2 * d, d, device="cuda")
    zst = torch.zeros(B, H, 2 * d, device="cuda")
    outs = []
    t = 0
    while t * min(Tc, F) < F:
        f0, w, cf, qf, ef = R.step_frames(t, F, Tc, To)
        sl_q, sl_k = slice(f0 * S, (f0 + qf) * S), slice(w * S, (f0 + qf) * S)
        outs.append(R.step_phi(qd[:, :, sl_q].contiguous(), kd[:, :, sl_k].contiguous(), vd[:, :, sl_k].contiguous(),
                               Pqd[:, :, sl_q].contiguous(), Pkd[:, :, sl_k].contiguous(), Sst, zst, S, qf, cf, ef))
        t += 1
    y = np64(torch.cat(outs, dim=2))
    ref = orc.oracle_recurrent(q, k, v, F, S, Tc, To, phi_q=Pq.double().numpy(), phi_k=Pk.double().numpy())
    assert_bf16_close(y, ref, "step_phi vs oracle")
    yf = np64(R.forward_phi(qd, kd, vd, Pqd, Pkd, F, S, Tc, To))
    assert np.linalg.norm(y - yf) / np.linalg.norm(yf) <= 5e-3


F32_TOL = 1e-5


@pytest.mark.parametrize("B,H,N,d,kind,seed", [(1, 2, 300, 128, "random", 60), (2, 1, 70, 64, "near_identity", 61)])
def test_phi_mlp_f32_matches_oracle(B, H, N, d, kind, seed):
    """The fp32 feature map against the oracle's fp64 MLP, relative L2 <= 1e-5."""
    x = inputs.make_qkv(B, H, N, d, seed, dtype="f32", scale=0.5)[0]
    w = tuple(t.float() for t in inputs.make_mlp_weights(H, d, seed, "q", kind))
    y = R.phi_mlp_f32(x.cuda(), *(t.cuda() for t in w)).cpu().double().numpy()
    ref = _oracle_phi(x, w)
    err = np.sqrt(((y - ref) ** 2).sum()) / np.sqrt((ref ** 2).sum())
    assert err <= F32_TOL, err


@pytest.mark.parametrize("F,S,Tc,To", [(4, 64, 2, 1), (5, 40, 2, 3), (6, 30, 3, 0)])
def test_forward_phi_f32_matches_oracle(F, S, Tc, To):
    """The fp32 learned-feature forward (fp32 feature map, then the fp32
    hybrid attention with those features) against the oracle end to end,
    relative L2 <= 1e-5 per (b, h)."""
    B, H, d = 1, 2, 64
    q, k, v = inputs.make_qkv(B, H, F * S, d, 62, dtype="f32", scale=0.5)
    wq = tuple(t.float() for t in inputs.make_mlp_weights(H, d, 62, "q", "random"))
    wk = tuple(t.float() for t in inputs.make_mlp_weights(H, d, 62, "k", "random"))
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    Pq = R.phi_mlp_f32(qd, *(t.cuda() for t in wq))
    Pk = R.phi_mlp_f32(kd, *(t.cuda() for t in wk))
    y = R.forward_phi_f32(qd, kd, vd, Pq, Pk, F, S, Tc, To).cpu().double().numpy()
    ref = orc.oracle_forward(q, k, v, F, S, Tc, To, phi_q=_oracle_phi(q, wq), phi_k=_oracle_phi(k, wk))
    num = np.sqrt(((y - ref) ** 2).sum(axis=(-2, -1)))
    den = np.sqrt((ref ** 2).sum(axis=(-2, -1)))
    assert (num / den).max() <= F32_TOL, (num / den).max()
