"""Where the bf16 path's error comes from, on the one skewed input whose
bf16 output cannot meet 3e-2 of the global RMS.

The fused kernel computes the softmax weights P = 2^(s log2(e)/sqrt(d) - m)
in fp32, rounds them to bf16 for the P.V tensor-core product (V is bf16, and
one MMA takes one operand type), sums exactly those bf16 weights into the
denominator, and moves the shift m lazily (only when a tile's maximum exceeds
it by more than 2^8), so that the accumulator in tensor memory is rescaled
rarely.  The output is rounded to bf16 at the end.

This file restates those rounding steps in numpy (no library call) on the
query-scaled balance input (q x 3, the sharpest softmax rows) and checks,
against the fp64 oracle:
  - that the emulation with bf16 weights lands above 3e-2 (the GPU measures
    the same figure, 3.23e-2, in tests/test_gpu_parity.py);
  - that with fp32 weights, or with an exact running shift (every weight of
    the row's largest key is then exactly 1), the error falls to the bf16
    rounding of the exact result itself, 2.71e-2;
so the excess is the bf16 rounding of the weights under the lazy shift, not
a mistake in the sets, the scale or the joint normaliser.
"""
import numpy as np
import torch

import oracle.rehyat_oracle as orc
from linear_attention_video_chunk_b200 import inputs

B, H, d, F, S, Tc, To = 1, 2, 128, 5, 160, 2, 1


def _bf16(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).bfloat16().double().numpy()


def _emulate(Q, K, V, h, bf16_weights=True, lazy=8.0):
    """The kernel's arithmetic for one head (fp32 scores, bf16 or fp32
    weights, lazy or exact shift, fixed phi linear term from exact states)."""
    N, Np, sl = F * S, Tc * S, np.log2(np.e) / np.sqrt(d)
    y = np.zeros((N, d))
    for t in range(-(-F // Tc)):
        q0, q1 = t * Np, min((t + 1) * Np, N)
        lo, hi = max(q0 - To * S, 0), q1
        s = (Q[h, q0:q1] @ K[h, lo:hi].T).astype(np.float32).astype(np.float64)
        m = np.zeros(q1 - q0) if lo > 0 else np.full(q1 - q0, -np.inf)
        O, l = np.zeros((q1 - q0, d)), np.zeros(q1 - q0)
        for j0 in range(0, hi - lo, 128):
            st = s[:, j0:j0 + 128]
            mx = st.max(1) * sl
            need = mx > m + lazy
            mnew = np.where(need, mx, m)
            alpha = np.where(need & np.isfinite(m), np.exp2(np.where(need, m - mnew, 0.0)), np.where(need, 0.0, 1.0))
            m = mnew
            O *= alpha[:, None]
            l *= alpha
            P = np.exp2(st * sl - m[:, None])
            if bf16_weights:
                P = _bf16(P)
            l += P.sum(1)
            O += P @ V[h, lo + j0:lo + j0 + st.shape[1]]
        if lo > 0:
            ph = _bf16(orc.phi(Q[h, q0:q1]) * np.exp2(-m)[:, None])
            PK = orc.phi(K[h, :lo])
            O += ph @ (PK.T @ V[h, :lo])
            l += ph @ PK.sum(0)
        y[q0:q1] = O / l[:, None]
    return y


def test_bf16_weights_under_the_lazy_shift_explain_the_sharp_input():
    q, k, v = inputs.make_qkv(B, H, F * S, d, 40, rms_qk=True, post=(3.0, 1.0, 1.0))
    ref = orc.oracle_forward(q, k, v, F, S, Tc, To)
    Q, K, V = (x[0].double().numpy() for x in (q, k, v))
    rms = np.sqrt((ref ** 2).mean())

    def out_err(**kw):
        y = np.stack([_emulate(Q, K, V, h, **kw) for h in range(H)])[None]
        return np.abs(_bf16(y) - ref).max() / rms

    floor = np.abs(_bf16(ref) - ref).max() / rms      # rounding the exact result
    assert 0.0270 < floor < 0.0272
    assert out_err() > 0.03                            # the kernel's roundings
    assert out_err(bf16_weights=False) <= floor + 1e-4  # fp32 weights: the floor
    assert out_err(lazy=0.0) <= floor + 1e-4            # exact shift: the floor
