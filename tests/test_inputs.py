"""Seeded input generator: determinism, per-head independence, rounding."""
import numpy as np
import torch

from linear_attention_video_chunk_b200 import inputs


def test_deterministic_and_per_head_streams():
    a = inputs.make_qkv(1, 3, 40, 16, seed=5)
    b = inputs.make_qkv(1, 3, 40, 16, seed=5)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    # a head can be regenerated alone
    h = inputs.head_array(5, "k", 0, 2, 40, 16)
    assert torch.equal(a[1][0, 2], torch.from_numpy(h.astype(np.float32)).to(torch.bfloat16))
    c = inputs.make_qkv(1, 3, 40, 16, seed=6)
    assert not torch.equal(a[0], c[0])


def test_rms_normalised_qk():
    q, k, v = inputs.make_qkv(1, 2, 64, 128, seed=1, rms_qk=True, dtype="f32")
    rms = q.pow(2).mean(-1).sqrt()
    assert torch.allclose(rms, torch.ones_like(rms), atol=1e-5)
    assert torch.allclose(k.pow(2).mean(-1).sqrt(), torch.ones_like(rms), atol=1e-5)
    assert abs(v.pow(2).mean().sqrt().item() - 1.0) < 0.05


def test_bf16_is_round_to_nearest_even():
    x = inputs.head_array(3, "q", 0, 0, 256, 64)
    got = inputs._store(x, "bf16").view(torch.int16).numpy().astype(np.uint16)
    f = x.astype(np.float32).view(np.uint32).astype(np.uint64)
    lsb = (f >> 16) & 1
    want = ((f + 0x7FFF + lsb) >> 16).astype(np.uint16)
    np.testing.assert_array_equal(got, want)


def test_mlp_weights_shapes_streams_and_kinds():
    """Learned-map stand-in weights: shapes and storage types the library
    takes, one stream per (seed, map, head), near-identity = the weights
    that make the MLP the fixed map plus small noise, random = no identity."""
    import oracle.rehyat_oracle as orc
    H, d = 3, 64
    W1, b1, W2, b2 = inputs.make_mlp_weights(H, d, 5, "q")
    assert (W1.shape, W2.shape, b1.shape, b2.shape) == ((H, 2 * d, d), (H, 2 * d, 2 * d), (H, 2 * d), (H, 2 * d))
    assert (W1.dtype, W2.dtype, b1.dtype, b2.dtype) == (torch.bfloat16, torch.bfloat16, torch.float32, torch.float32)
    again = inputs.make_mlp_weights(H, d, 5, "q")
    assert all(torch.equal(a, b) for a, b in zip((W1, b1, W2, b2), again))
    Wk = inputs.make_mlp_weights(H, d, 5, "k")[0]
    assert not torch.equal(W1, Wk) and not torch.equal(W1[0], W1[1])
    I1, _, I2, _ = orc.mlp_identity_weights(d)
    dev1 = (W1.double().numpy() - I1).std()
    dev2 = (W2.double().numpy() - I2).std()
    assert 0.05 / d ** 0.5 < dev1 < 0.2 / d ** 0.5 and 0.05 / (2 * d) ** 0.5 < dev2 < 0.2 / (2 * d) ** 0.5
    assert float(b1.abs().max()) < 0.1 and float(b2.abs().max()) < 0.1
    R1 = inputs.make_mlp_weights(H, d, 5, "q", kind="random")[0].double().numpy()
    assert abs(R1.std() - 1 / d ** 0.5) < 0.1 / d ** 0.5 and abs((R1 - I1).mean()) < 0.05
