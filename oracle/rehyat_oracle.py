"""Plain fp64 CPU oracle for ReHyAt's temporally chunked hybrid attention.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py`` (its ``cpu_baseline`` leg and its
``--impl reference`` arm) may import or call anything in this package.  The
CUDA library never imports it, and this module imports nothing from the CUDA
package: the two share no code.  Every function is written straight from the
equations of "ReHyAt: Recurrent Hybrid Attention for Video Diffusion
Transformers" (Ghafoorian & Habibian, arXiv 2601.04342); the section / equation
each one follows is named in its docstring.  Everything is float64 numpy; the
inputs are the exact values the GPU sees (bf16- or fp32-rounded, then widened).

Notation (the paper's):
  HW      tokens per latent frame           (library name: S_tok)
  T_c     frames per temporal chunk         (chunk_frames)
  T_o     overlap frames                    (overlap_frames)
  N'      tokens per chunk = T_c * HW       (reading R2: the paper never defines N')
  N       tokens in the video = F * HW, frame-major order j = f*HW + spatial index
  phi     feature map, D' = 2d  (P = 2, psi_1 = psi_2 = 1 + elu; reading R5)

Set modes:
  "causal"        §3.3 (Recurrent HyAt) sets: T^L_t = {j < lo_t},
                  T^S_t = {lo_t <= j < (t+1)N'}, lo_t = max(tN' - T_o HW, 0).
                  This is what rehyat_forward / rehyat_step compute.
  "bidirectional" §3.2 sets with overlap: same T^S_t, T^L_t = T - T^S_t.
                  (With T_o = 0 these are the §3.2 sets without overlap.)
  "linear_only"   test-only: T^S = {} and T^L = T for every query, so the hybrid
                  reduces to the §3.1 linear-attention equation.

Parity status: every function here is pinned by tests/test_oracle_pins.py
(closed forms, hand-derived worked examples in tests/golden/, library
reductions and brute force); none is "parity unpinned".
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "psi", "phi", "phi_mlp", "mlp_identity_weights", "n_chunks", "chunk_geometry", "hybrid_mask_rows",
    "oracle_parts", "oracle_forward", "oracle_recurrent", "oracle_bruteforce",
    "oracle_chunk_states", "oracle_step",
]

MODES = ("causal", "bidirectional", "linear_only")


# --------------------------------------------------------------------------- #
# Feature map                                                                  #
# --------------------------------------------------------------------------- #
def psi(x):
    """psi(x) = 1 + elu(x): x + 1 for x > 0, exp(x) for x <= 0.

    §3.1 gives 1 + elu (Katharopoulos et al.) as the non-negative map the
    linear kernel needs; reading R5 uses it for both polynomial terms of §3.2.
    """
    x = np.asarray(x, dtype=np.float64)
    return np.where(x > 0.0, x + 1.0, np.exp(np.minimum(x, 0.0)))


def phi(x):
    """§3.2 polynomial feature map phi(x) = [psi_1(x)^1, psi_2(x)^2] with P = 2.

    Applied to the last axis (length d); returns length D' = 2d with the first
    d features psi(x) and the last d features psi(x)**2.
    """
    p = psi(x)
    return np.concatenate([p, p * p], axis=-1)


def phi_mlp(x, W1, b1, W2, b2):
    """Learned feature map ("ReHyAt", §4.3 Training specification and §7.1
    Training Details): a two-layer MLP with degree-2 polynomial features,
    phi(x) = [psi_1(x)^1, psi_2(x)^2] (the §3.2 feature-map equation, P = 2).
    The paper fixes neither the hidden width nor the output non-linearity; the
    reading taken here is hidden width 2d and psi_p = 1 + elu of the MLP
    outputs, which keeps phi non-negative (§3.1) and gives the paper's
    parameter count.

      h     = relu(W1 x + b1)             W1: [2d, d], b1: [2d]  (hidden 2d)
      u     = W2 h + b2                   W2: [2d, 2d], b2: [2d]
      psi_p = 1 + elu(u_p)                u_1 = u[:d], u_2 = u[d:]
      phi   = [psi_1, psi_2 ** 2]         (non-negative, §3.1)

    Per head and per map (q or k): 2d*d + 2d*2d = 98,304 weights at d = 128,
    i.e. 2.36 M for the 12 heads of a block and both maps (the paper: about
    2.4 M per converted block).  x: [..., d] -> [..., 2d] (float64).
    """
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    h = np.maximum(x @ np.asarray(W1, dtype=np.float64).T + np.asarray(b1, dtype=np.float64), 0.0)
    u = h @ np.asarray(W2, dtype=np.float64).T + np.asarray(b2, dtype=np.float64)
    p1 = psi(u[..., :d])
    p2 = psi(u[..., d:])
    return np.concatenate([p1, p2 * p2], axis=-1)


def mlp_identity_weights(d):
    """Weights with which phi_mlp is exactly the fixed map phi: the hidden
    layer holds relu(x) and relu(-x) (W1 = [I; -I]) and each output block
    recombines them to x (W2 rows [I, -I]), so u_1 = u_2 = x."""
    I = np.eye(d)
    W1 = np.concatenate([I, -I], axis=0)
    W2 = np.concatenate([np.concatenate([I, -I], axis=1)] * 2, axis=0)
    return W1, np.zeros(2 * d), W2, np.zeros(2 * d)


# --------------------------------------------------------------------------- #
# Chunk geometry and the explicit hybrid mask                                  #
# --------------------------------------------------------------------------- #
def n_chunks(F: int, T_c: int) -> int:
    """Number of temporal chunks: ceil(F / T_c) (reading R4: last one ragged)."""
    return -(-F // T_c)


def chunk_geometry(t: int, F: int, HW: int, T_c: int, T_o: int):
    """Token ranges of chunk t: (q0, q1, lo, hi).

    Queries of chunk t are [q0, q1) = [tN', min((t+1)N', N)) (reading R8: each
    query belongs to exactly one chunk).  Its softmax set is [lo, hi) with
    lo = max(tN' - T_o HW, 0) and hi = min((t+1)N', N) (§3.2 / §3.3 sets,
    clipped to T = [0, N) per reading R4).
    """
    N = F * HW
    Np = T_c * HW
    q0 = t * Np
    q1 = min((t + 1) * Np, N)
    lo = max(t * Np - T_o * HW, 0)
    return q0, q1, lo, q1


def hybrid_mask_rows(rows, F: int, HW: int, T_c: int, T_o: int, mode: str = "causal"):
    """Rows of the explicit N x N hybrid mask for the given query indices.

    Returns (in_S, in_L): boolean arrays [len(rows), N]; in_S[r, j] says key j
    is in T^S_t of query rows[r], in_L[r, j] that it is in T^L_t.  For small N
    pass rows = range(N) to get the full mask.
    """
    if mode not in MODES:
        raise ValueError(f"unknown mode {mode!r}")
    N = F * HW
    Np = T_c * HW
    rows = np.asarray(rows, dtype=np.int64)
    t = rows // Np
    j = np.arange(N, dtype=np.int64)[None, :]
    lo = np.maximum(t * Np - T_o * HW, 0)[:, None]
    hi = np.minimum((t + 1) * Np, N)[:, None]
    in_S = (j >= lo) & (j < hi)
    if mode == "causal":
        in_L = j < lo
    elif mode == "bidirectional":
        in_L = ~in_S
    else:  # linear_only
        in_S = np.zeros((rows.size, N), dtype=bool)
        in_L = np.ones((rows.size, N), dtype=bool)
    return in_S, in_L


def _f64(x):
    if hasattr(x, "detach"):  # torch tensor
        x = x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def _features(f, X, idx, b, h):
    """phi of the rows idx of X (one head): f is a per-head map f(x, h), or an
    array [B, H, N, D'] of precomputed features indexed by (b, h, row)."""
    if callable(f):
        return f(X[idx], h)
    return np.asarray(f, dtype=np.float64)[b, h][idx]


# --------------------------------------------------------------------------- #
# Parallel form, explicit mask                                                 #
# --------------------------------------------------------------------------- #
def oracle_parts(q, k, v, F, HW, T_c, T_o, mode="causal", rows=None, block=512, phi_q=None, phi_k=None):
    """The four unnormalised terms of the §3.2 joint normaliser, per query.

    For each (b, h) and query i of chunk t:
      a^S_i = sum_{j in T^S_t} exp(q_i.k_j / sqrt(d)) v_j     n^S_i = sum exp(...)
      a^L_i = sum_{j in T^L_t} (phi(q_i).phi(k_j)) v_j         n^L_i = sum phi.phi
    computed pairwise from the explicit mask rows (never through the cached
    sums of §3.1).  Softmax scale 1/sqrt(d) is reading R6.  No max shift: in
    fp64 the scores of these workloads are far from overflow, and a non-finite
    result raises.

    q, k, v: [B, H, N, d].  rows: optional query indices (all if None).
    phi_q / phi_k: optional per-head feature maps, callables f(x, h) -> phi,
    or arrays [B, H, N, D'] of precomputed features (default: the fixed phi).
    Returns aS [B,H,R,d], nS [B,H,R], aL [B,H,R,d], nL [B,H,R] (float64).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, d = q.shape
    assert N == F * HW, "N must equal F * HW"
    rows = np.arange(N) if rows is None else np.asarray(rows, dtype=np.int64)
    R = rows.size
    aS = np.zeros((B, H, R, d))
    aL = np.zeros((B, H, R, d))
    nS = np.zeros((B, H, R))
    nL = np.zeros((B, H, R))
    scale = 1.0 / math.sqrt(d)
    fq = phi_q if phi_q is not None else (lambda x, h: phi(x))
    fk = phi_k if phi_k is not None else (lambda x, h: phi(x))
    for b in range(B):
        for h in range(H):
            Q, K, V = q[b, h], k[b, h], v[b, h]
            phiK = _features(fk, K, slice(None), b, h)
            for r0 in range(0, R, block):
                rb = rows[r0:r0 + block]
                in_S, in_L = hybrid_mask_rows(rb, F, HW, T_c, T_o, mode)
                s = (Q[rb] @ K.T) * scale
                wS = np.exp(np.where(in_S, s, -np.inf))
                wL = np.where(in_L, _features(fq, Q, rb, b, h) @ phiK.T, 0.0)
                aS[b, h, r0:r0 + rb.size] = wS @ V
                nS[b, h, r0:r0 + rb.size] = wS.sum(axis=1)
                aL[b, h, r0:r0 + rb.size] = wL @ V
                nL[b, h, r0:r0 + rb.size] = wL.sum(axis=1)
    if not (np.isfinite(aS).all() and np.isfinite(nS).all()):
        raise FloatingPointError("softmax term overflowed in fp64")
    return aS, nS, aL, nL


def oracle_forward(q, k, v, F, HW, T_c, T_o, mode="causal", rows=None, block=512, phi_q=None, phi_k=None):
    """Hybrid attention output y_i = (a^S + a^L) / (n^S + n^L)  (§3.2 joint
    normalisation), with the sets of ``mode``.  Returns [B, H, R, d] float64."""
    aS, nS, aL, nL = oracle_parts(q, k, v, F, HW, T_c, T_o, mode, rows, block, phi_q, phi_k)
    return (aS + aL) / (nS + nL)[..., None]


# --------------------------------------------------------------------------- #
# Chunk-wise recurrent form                                                    #
# --------------------------------------------------------------------------- #
def oracle_chunk_states(k, v, F, HW, T_c, T_o):
    """Linear-attention state entering each chunk under the §3.3 sets.

    S_t = sum_{j < lo_t} phi(k_j) v_j^T  (D' x d) and z_t = sum_{j < lo_t}
    phi(k_j)  (D'), i.e. the two sums §3.1 notes are independent of the query,
    restricted to T^L_t.  Returns S [B,H,n_chunks,D',d], z [B,H,n_chunks,D'].
    """
    k, v = _f64(k), _f64(v)
    B, H, N, d = k.shape
    nc = n_chunks(F, T_c)
    S = np.zeros((B, H, nc, 2 * d, d))
    z = np.zeros((B, H, nc, 2 * d))
    for t in range(nc):
        _, _, lo, _ = chunk_geometry(t, F, HW, T_c, T_o)
        pk = phi(k[:, :, :lo])                         # [B,H,lo,D']
        S[:, :, t] = np.einsum("bhje,bhjc->bhec", pk, v[:, :, :lo])
        z[:, :, t] = pk.sum(axis=2)
    return S, z


def oracle_recurrent(q, k, v, F, HW, T_c, T_o, phi_q=None, phi_k=None):
    """§3.3 chunk-wise RNN: walk the chunks in order with a constant-size state.

    Before chunk t the state (S, z) is advanced by folding in the keys
    [folded, lo_t) that have left every later softmax window; the chunk's
    queries then take exact softmax over [lo_t, hi_t) plus phi(q) S and
    phi(q) z (the §3.1 caching argument), jointly normalised (§3.2).
    Returns [B, H, N, d] float64.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, d = q.shape
    out = np.zeros_like(q)
    scale = 1.0 / math.sqrt(d)
    fq = phi_q if phi_q is not None else (lambda x, h: phi(x))
    fk = phi_k if phi_k is not None else (lambda x, h: phi(x))
    for b in range(B):
        for h in range(H):
            Q, K, V = q[b, h], k[b, h], v[b, h]
            S = np.zeros((2 * d, d))
            z = np.zeros(2 * d)
            folded = 0
            for t in range(n_chunks(F, T_c)):
                q0, q1, lo, hi = chunk_geometry(t, F, HW, T_c, T_o)
                pk = _features(fk, K, slice(folded, lo), b, h)
                S = S + pk.T @ V[folded:lo]
                z = z + pk.sum(axis=0)
                folded = lo
                e = np.exp((Q[q0:q1] @ K[lo:hi].T) * scale)
                pq = _features(fq, Q, slice(q0, q1), b, h)
                num = e @ V[lo:hi] + pq @ S
                den = e.sum(axis=1) + pq @ z
                out[b, h, q0:q1] = num / den[:, None]
    return out


def oracle_step(q_c, k_c, v_c, S, z, HW, evict_frames):
    """One step of the §3.3 recurrent form as the library's step call frames it.

    q_c [B,H,Lq,d] are the chunk's queries, k_c / v_c [B,H,Lk,d] its whole
    softmax window (overlap frames then the chunk's own frames), S [B,H,D',d]
    and z [B,H,D'] the state of all earlier keys.  Output = (softmax over the
    window + phi(q) S) / (softmax mass + phi(q) z); afterwards the first
    evict_frames * HW window keys are folded into the state.
    Returns (out [B,H,Lq,d], S', z') in float64.
    """
    q_c, k_c, v_c, S, z = map(_f64, (q_c, k_c, v_c, S, z))
    d = q_c.shape[-1]
    s = np.einsum("bhid,bhjd->bhij", q_c, k_c) / math.sqrt(d)
    e = np.exp(s)
    pq = phi(q_c)
    num = np.einsum("bhij,bhjd->bhid", e, v_c) + np.einsum("bhie,bhed->bhid", pq, S)
    den = e.sum(axis=-1) + np.einsum("bhie,bhe->bhi", pq, z)
    out = num / den[..., None]
    ne = evict_frames * HW
    pk = phi(k_c[:, :, :ne])
    S2 = S + np.einsum("bhje,bhjd->bhed", pk, v_c[:, :, :ne])
    z2 = z + pk.sum(axis=2)
    return out, S2, z2


# --------------------------------------------------------------------------- #
# Brute force (pure Python, tiny inputs only)                                  #
# --------------------------------------------------------------------------- #
def oracle_bruteforce(q, k, v, F, HW, T_c, T_o, mode="causal", phi_q=None, phi_k=None):
    """Double loop over (query, key) pairs with set membership decided inline
    from the §3.2 / §3.3 set definitions: no mask matrix, no numpy algebra.
    Intended for N <= ~64 and d <= ~8.  Returns nested lists [B][H][N][d].

    phi_q / phi_k: optional per-vector feature maps f(x, h) -> sequence of
    D' floats; the linear weight is then their dot product, summed in a loop
    (default: the fixed phi, inline per element)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, d = q.shape
    Np = T_c * HW
    rs = 1.0 / math.sqrt(d)

    def psi1(x):
        return x + 1.0 if x > 0.0 else math.exp(x)

    out = []
    for b in range(B):
        ob = []
        for h in range(H):
            oh = []
            for i in range(N):
                t = i // Np
                lo = max(t * Np - T_o * HW, 0)
                hi = min((t + 1) * Np, N)
                num = [0.0] * d
                den = 0.0
                for j in range(N):
                    local = lo <= j < hi
                    if mode == "linear_only":
                        local, glob = False, True
                    elif mode == "causal":
                        glob = j < lo
                    else:
                        glob = not local
                    if local:
                        dot = 0.0
                        for c in range(d):
                            dot += q[b, h, i, c] * k[b, h, j, c]
                        w = math.exp(dot * rs)
                    elif glob and phi_q is not None:
                        fa = list(phi_q(q[b, h, i], h))
                        fb = list(phi_k(k[b, h, j], h))
                        w = 0.0
                        for e in range(len(fa)):
                            w += fa[e] * fb[e]
                    elif glob:
                        w = 0.0
                        for c in range(d):
                            a = psi1(q[b, h, i, c])
                            bb = psi1(k[b, h, j, c])
                            w += a * bb + (a * a) * (bb * bb)
                    else:
                        continue
                    for c in range(d):
                        num[c] += w * v[b, h, j, c]
                    den += w
                oh.append([x / den for x in num])
            ob.append(oh)
        out.append(ob)
    return out
