"""Seeded synthetic inputs shared by the tests, the bench and the oracle checks.

This module holds no arithmetic of the attention method: it only draws Gaussian
Q/K/V, optionally RMS-normalises Q and K per head vector (the stand-in for the
Wan2.1 QK-RMSNorm that precedes attention in the target DiTs), and rounds to
the storage dtype.  Both the CUDA path and the oracle consume its output.

Recipe (one independent numpy PCG64 stream per tensor and head, so any head can
be regenerated alone for sampled-row checks):
  stream(seed, which, b, h) = default_rng(SeedSequence([seed, which, b, h]))
  which: 0 = q, 1 = k, 2 = v;  x = scale * standard_normal((N, d)) in float64
  rms_qk: q, k -> x / sqrt(mean(x**2, axis=-1) + 1e-6)
  post:   optional per-tensor factors applied after the RMS step (to make the
          softmax branch dominate, or the linear one, in targeted tests)
  storage: float32, then bfloat16 by round-to-nearest-even (torch's cast).
Heads are generated in parallel threads; the result does not depend on that.

Learned feature-map weights (make_mlp_weights; the trained weights of the
paper are not available, so they are drawn): per map (q or k) and head,
  stream = default_rng(SeedSequence([seed, 10 + which, h]))
  "near_identity": W1 = [I; -I] + noise/sqrt(d), W2 = [[I, -I]; [I, -I]]
                   + noise/sqrt(2d) (the weights with which the map is the
                   fixed 1 + elu features, the natural start of a
                   distillation), biases noise * 0.1 * N(0, 1)
  "random":        W1 = N(0,1)/sqrt(d), W2 = N(0,1)/sqrt(2d), biases 0.1 N(0,1)
  W1, W2 stored bf16, b1, b2 fp32.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

WHICH = {"q": 0, "k": 1, "v": 2}


def head_array(seed: int, which: str, b: int, h: int, N: int, d: int,
               scale: float = 1.0, rms_qk: bool = False, post: float = 1.0) -> np.ndarray:
    """float64 [N, d] draw for one (tensor, batch, head)."""
    rng = np.random.default_rng(np.random.SeedSequence([seed, WHICH[which], b, h]))
    x = rng.standard_normal((N, d)) * scale
    if rms_qk and which in ("q", "k"):
        x = x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + 1e-6)
    return x * post if post != 1.0 else x


def _store(x64: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(x64.astype(np.float32))
    if dtype == "bf16":
        return t.to(torch.bfloat16)
    if dtype == "f32":
        return t
    raise ValueError(dtype)


def make_qkv(B: int, H: int, N: int, d: int, seed: int, dtype: str = "bf16",
             scale: float = 1.0, rms_qk: bool = False, post=(1.0, 1.0, 1.0), pin: bool = False):
    """Host tensors q, k, v of shape [B, H, N, d] in the storage dtype.

    scale multiplies the N(0,1) draw; post = (sq, sk, sv) multiplies each
    tensor after the optional RMS normalisation.  pin: page-locked memory.
    """
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    out = [torch.empty((B, H, N, d), dtype=tdt, pin_memory=pin) for _ in range(3)]
    jobs = [(i, which, b, h) for i, which in enumerate(("q", "k", "v")) for b in range(B) for h in range(H)]

    def fill(job):
        i, which, b, h = job
        out[i][b, h] = _store(head_array(seed, which, b, h, N, d, scale, rms_qk, post[i]), dtype)

    workers = max(1, min(len(jobs), len(os.sched_getaffinity(0))))
    with ThreadPoolExecutor(workers) as ex:
        list(ex.map(fill, jobs))
    return tuple(out)


def make_state(B: int, H: int, d: int, seed: int, scale: float = 1.0):
    """A non-negative z and arbitrary S, fp32, shaped like a recurrent state
    ([B,H,2d,d], [B,H,2d]); used only to exercise the step call from a
    non-zero starting state."""
    rng = np.random.default_rng(np.random.SeedSequence([seed, 7]))
    S = rng.standard_normal((B, H, 2 * d, d)) * scale
    z = np.abs(rng.standard_normal((B, H, 2 * d))) * scale + 1.0
    return torch.from_numpy(S.astype(np.float32)), torch.from_numpy(z.astype(np.float32))


def make_mlp_weights(H: int, d: int, seed: int, which: str = "q", kind: str = "near_identity",
                     noise: float = 0.1):
    """Host (W1 [H,2d,d] bf16, b1 [H,2d] fp32, W2 [H,2d,2d] bf16, b2 [H,2d] fp32)."""
    W1 = np.empty((H, 2 * d, d))
    W2 = np.empty((H, 2 * d, 2 * d))
    b1 = np.empty((H, 2 * d))
    b2 = np.empty((H, 2 * d))
    I = np.eye(d)
    for h in range(H):
        rng = np.random.default_rng(np.random.SeedSequence([seed, 10 + WHICH[which], h]))
        n1 = rng.standard_normal((2 * d, d)) / np.sqrt(d)
        n2 = rng.standard_normal((2 * d, 2 * d)) / np.sqrt(2 * d)
        c1 = rng.standard_normal(2 * d) * 0.1
        c2 = rng.standard_normal(2 * d) * 0.1
        if kind == "near_identity":
            W1[h] = np.concatenate([I, -I], axis=0) + noise * n1
            W2[h] = np.concatenate([np.concatenate([I, -I], axis=1)] * 2, axis=0) + noise * n2
            b1[h], b2[h] = noise * c1, noise * c2
        elif kind == "random":
            W1[h], W2[h], b1[h], b2[h] = n1, n2, c1, c2
        else:
            raise ValueError(kind)
    return (_store(W1, "bf16"), torch.from_numpy(b1.astype(np.float32)), _store(W2, "bf16"),
            torch.from_numpy(b2.astype(np.float32)))
