"""ctypes binding of librehyat.so (the C ABI in include/rehyat.h).

Argument marshalling only: every step of the computation runs in the
library's CUDA kernels.  Tensors are torch CUDA tensors (used for device
memory); calls go on torch's current stream.  There is no CPU fallback: if the
library is missing or a call fails, a RuntimeError is raised.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librehyat.so")

_c_int, _c_size, _vp, _fp = ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_void_p
_I = _c_int

# name -> argtypes (all return int unless listed in _RESTYPES)
_SIGS = {
    "rehyat_status_string": [_I],
    "rehyat_forward": [_vp, _vp, _vp, _I, _I, _I, _I, _I, _I, _I, _vp, _vp],
    "rehyat_forward_workspace_bytes": [_I, _I, _I, _I, _I, _I, _I, ctypes.POINTER(_c_size)],
    "rehyat_forward_ws": [_vp, _vp, _vp, _I, _I, _I, _I, _I, _I, _I, _vp, _vp, _c_size, _vp],
    "rehyat_forward_states": [_vp, _vp, _I, _I, _I, _I, _I, _I, _I, _vp, _c_size, _vp],
    "rehyat_forward_attention": [_vp, _vp, _vp, _I, _I, _I, _I, _I, _I, _I, _vp, _vp, _c_size, _vp],
    "rehyat_forward_f32": [_vp, _vp, _vp, _I, _I, _I, _I, _I, _I, _I, _vp, _vp],
    "rehyat_forward_parts": [_vp, _vp, _vp, _I, _I, _I, _I, _I, _I, _I, _vp, _vp, _vp, _vp, _vp, _vp],
    "rehyat_chunk_states": [_vp, _vp, _I, _I, _I, _I, _I, _I, _I, _vp, _vp, _vp],
    "rehyat_step": [_vp, _vp, _vp, _vp, _vp, _vp, _I, _I, _I, _I, _I, _I, _I, _vp],
    "rehyat_step_workspace_bytes": [_I, _I, _I, _I, _I, _I, _I, ctypes.POINTER(_c_size)],
    "rehyat_step_ws": [_vp, _vp, _vp, _vp, _vp, _vp, _I, _I, _I, _I, _I, _I, _I, _vp, _c_size, _vp],
    "rehyat_step_f32": [_vp, _vp, _vp, _vp, _vp, _vp, _I, _I, _I, _I, _I, _I, _I, _vp],
    "rehyat_phi": [_vp, _I, _vp, _I, ctypes.c_int64, _I, _vp],
    "rehyat_device_status": [ctypes.POINTER(ctypes.c_uint)],
    "rehyat_forward_noalloc": [_vp, _vp, _vp, _I, _I, _I, _I, _I, _I, _I, _vp, _vp],
    "rehyat_forward_ex_workspace_bytes": [_I, _I, _I, _I, _I, _I, _I, _I, ctypes.POINTER(_c_size)],
    "rehyat_forward_ex": [_vp, _vp, _vp, _I, _I, _I, _I, _I, _I, _I, _I, _I, _vp, _vp, _c_size, _vp],
    "rehyat_phi_mlp": [_vp, _I, _I, _I, _I, _I, _vp, _vp, _vp, _vp, _vp, _vp],
    "rehyat_forward_phi": [_vp, _vp, _vp, _vp, _vp, _I, _I, _I, _I, _I, _I, _I, _I, _I, _vp, _vp, _c_size, _vp],
    "rehyat_forward_mlp_workspace_bytes": [_I, _I, _I, _I, _I, _I, _I, _I, ctypes.POINTER(_c_size)],
    "rehyat_forward_mlp": [_vp] * 11 + [_I] * 9 + [_vp, _vp, _c_size, _vp],
    "rehyat_step_phi": [_vp] * 8 + [_I] * 7 + [_vp, _c_size, _vp],
    "rehyat_forward_host_workspace_bytes": [_I, _I, _I, _I, _I, _I, _I, _I, ctypes.POINTER(_c_size)],
    "rehyat_forward_host": [_vp, _vp, _vp] + [_I] * 9 + [_vp, _vp, _c_size, _vp],
    "rehyat_phi_mlp_f32": [_vp, _I, _I, _I, _I, _vp, _vp, _vp, _vp, _vp, _vp],
    "rehyat_step_ex": [_vp] * 6 + [_I] * 8 + [_vp, _c_size, _vp],
    "rehyat_wait_probe": [_vp, _vp],
    "rehyat_forward_phi_f32": [_vp] * 5 + [_I] * 7 + [_vp, _vp],
}
_RESTYPES = {"rehyat_status_string": ctypes.c_char_p}

OK, EINVAL, EUNSUPPORTED, ENOMEM, ECUDA, ETIMEOUT = range(6)
SETS = {"causal": 0, "bidirectional": 1}
LAYOUTS = {"bhnd": 0, "bnhd": 1}
DTYPE_BF16, DTYPE_F32 = 0, 1

_lib = None


class RehyatError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


def lib() -> ctypes.CDLL:
    """Load librehyat.so (once).  Raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing; build it with `python -m linear_attention_video_chunk_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, args in _SIGS.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = _RESTYPES.get(name, _c_int)
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().rehyat_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != OK:
        raise RehyatError(status, where)


def _p(t):
    return _vp(t.data_ptr()) if t is not None else _vp(0)


def _stream():
    return _vp(torch.cuda.current_stream().cuda_stream)


def _need(t: torch.Tensor, dtype, name: str, ndim: int = 4):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims")


def _shape(q, F, S_tok):
    B, H, N, d = q.shape
    if N != F * S_tok:
        raise ValueError(f"N={N} != F*S_tok={F * S_tok}")
    return B, H, N, d


# --------------------------------------------------------------------------- #
# parallel form                                                                #
# --------------------------------------------------------------------------- #
def workspace_bytes(B, H, F, S_tok, d, chunk_frames, overlap_frames) -> int:
    n = _c_size(0)
    _check(lib().rehyat_forward_workspace_bytes(B, H, F, S_tok, d, chunk_frames, overlap_frames, ctypes.byref(n)),
           "rehyat_forward_workspace_bytes")
    return n.value


def alloc_workspace(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def forward(q, k, v, F, S_tok, chunk_frames, overlap_frames, out=None, workspace=None):
    """bf16 hybrid attention forward (parallel form) -> out [B,H,N,d] bf16.

    Scratch comes from torch's caching allocator (or ``workspace``) and is
    passed to rehyat_forward_ws."""
    for n, t in (("q", q), ("k", k), ("v", v)):
        _need(t, torch.bfloat16, n)
    B, H, N, d = _shape(q, F, S_tok)
    out = torch.empty_like(q) if out is None else out
    _need(out, torch.bfloat16, "out")
    nb = workspace_bytes(B, H, F, S_tok, d, chunk_frames, overlap_frames)
    ws = alloc_workspace(nb, q.device) if workspace is None else workspace
    _check(lib().rehyat_forward_ws(_p(q), _p(k), _p(v), B, H, F, S_tok, d, chunk_frames, overlap_frames, _p(out),
                                   _p(ws), ws.numel(), _stream()), "rehyat_forward_ws")
    return out


def forward_sets(q, k, v, F, S_tok, chunk_frames, overlap_frames, sets="causal", layout="bhnd", out=None,
                 workspace=None):
    """rehyat_forward_ex: the forward with the "causal" (§3.3, default) or
    "bidirectional" (§3.2, non-causal) sets, on [B,H,N,d] ("bhnd") or
    [B,N,H,d] ("bnhd") tensors."""
    for n, t in (("q", q), ("k", k), ("v", v)):
        _need(t, torch.bfloat16, n)
    if layout == "bhnd":
        B, H, N, d = _shape(q, F, S_tok)
    else:
        B, N, H, d = q.shape
        if N != F * S_tok:
            raise ValueError(f"N={N} != F*S_tok={F * S_tok}")
    out = torch.empty_like(q) if out is None else out
    n = _c_size(0)
    _check(lib().rehyat_forward_ex_workspace_bytes(B, H, F, S_tok, d, chunk_frames, overlap_frames, SETS[sets],
                                                   ctypes.byref(n)), "rehyat_forward_ex_workspace_bytes")
    ws = alloc_workspace(n.value, q.device) if workspace is None else workspace
    _check(lib().rehyat_forward_ex(_p(q), _p(k), _p(v), B, H, F, S_tok, d, chunk_frames, overlap_frames, SETS[sets],
                                   LAYOUTS[layout], _p(out), _p(ws), ws.numel(), _stream()), "rehyat_forward_ex")
    return out


def _dims(q, F, S_tok, layout):
    if layout == "bhnd":
        return _shape(q, F, S_tok)
    B, N, H, d = q.shape
    if N != F * S_tok:
        raise ValueError(f"N={N} != F*S_tok={F * S_tok}")
    return B, H, N, d


def _need_mlp(w, H, d, name):
    """w = (W1 [H,2d,d] bf16, b1 [H,2d] fp32, W2 [H,2d,2d] bf16, b2 [H,2d] fp32)."""
    if len(w) != 4:
        raise ValueError(f"{name} must be (W1, b1, W2, b2)")
    W1, b1, W2, b2 = w
    for n, t, dt, shape in (("W1", W1, torch.bfloat16, (H, 2 * d, d)), ("b1", b1, torch.float32, (H, 2 * d)),
                            ("W2", W2, torch.bfloat16, (H, 2 * d, 2 * d)), ("b2", b2, torch.float32, (H, 2 * d))):
        _need(t, dt, f"{name}.{n}", len(shape))
        if tuple(t.shape) != shape:
            raise ValueError(f"{name}.{n} must be {shape}, got {tuple(t.shape)}")
    return W1, b1, W2, b2


def phi_mlp(x, W1, b1, W2, b2, layout="bhnd", out=None):
    """rehyat_phi_mlp: learned feature map of x ([B,H,N,d] or [B,N,H,d] bf16)
    with per-head weights -> phi [B,H,N,2d] bf16."""
    _need(x, torch.bfloat16, "x")
    if layout == "bhnd":
        B, H, N, d = x.shape
    else:
        B, N, H, d = x.shape
    _need_mlp((W1, b1, W2, b2), H, d, "weights")
    out = torch.empty((B, H, N, 2 * d), dtype=torch.bfloat16, device=x.device) if out is None else out
    _need(out, torch.bfloat16, "out")
    _check(lib().rehyat_phi_mlp(_p(x), B, H, N, d, LAYOUTS[layout], _p(W1), _p(b1), _p(W2), _p(b2), _p(out),
                                _stream()), "rehyat_phi_mlp")
    return out


def forward_phi(q, k, v, phi_q, phi_k, F, S_tok, chunk_frames, overlap_frames, sets="causal", layout="bhnd",
                out=None, workspace=None):
    """rehyat_forward_phi: the forward with precomputed feature maps phi_q,
    phi_k ([B,H,N,2d] bf16, non-negative) in the linear term and states."""
    for n, t in (("q", q), ("k", k), ("v", v), ("phi_q", phi_q), ("phi_k", phi_k)):
        _need(t, torch.bfloat16, n)
    B, H, N, d = _dims(q, F, S_tok, layout)
    for n, t in (("phi_q", phi_q), ("phi_k", phi_k)):
        if tuple(t.shape) != (B, H, N, 2 * d):
            raise ValueError(f"{n} must be {(B, H, N, 2 * d)}")
    out = torch.empty_like(q) if out is None else out
    n = _c_size(0)
    _check(lib().rehyat_forward_ex_workspace_bytes(B, H, F, S_tok, d, chunk_frames, overlap_frames, SETS[sets],
                                                   ctypes.byref(n)), "rehyat_forward_ex_workspace_bytes")
    ws = alloc_workspace(n.value, q.device) if workspace is None else workspace
    _check(lib().rehyat_forward_phi(_p(q), _p(k), _p(v), _p(phi_q), _p(phi_k), B, H, F, S_tok, d, chunk_frames,
                                    overlap_frames, SETS[sets], LAYOUTS[layout], _p(out), _p(ws), ws.numel(),
                                    _stream()), "rehyat_forward_phi")
    return out


def forward_mlp_workspace_bytes(B, H, F, S_tok, d, chunk_frames, overlap_frames, sets="causal") -> int:
    n = _c_size(0)
    _check(lib().rehyat_forward_mlp_workspace_bytes(B, H, F, S_tok, d, chunk_frames, overlap_frames, SETS[sets],
                                                    ctypes.byref(n)), "rehyat_forward_mlp_workspace_bytes")
    return n.value


def forward_mlp(q, k, v, wq, wk, F, S_tok, chunk_frames, overlap_frames, sets="causal", layout="bhnd", out=None,
                workspace=None):
    """rehyat_forward_mlp: learned phi_q (weights wq) and phi_k (wk), each
    (W1, b1, W2, b2), then the hybrid forward."""
    for n, t in (("q", q), ("k", k), ("v", v)):
        _need(t, torch.bfloat16, n)
    B, H, N, d = _dims(q, F, S_tok, layout)
    Wq1, bq1, Wq2, bq2 = _need_mlp(wq, H, d, "wq")
    Wk1, bk1, Wk2, bk2 = _need_mlp(wk, H, d, "wk")
    out = torch.empty_like(q) if out is None else out
    nb = forward_mlp_workspace_bytes(B, H, F, S_tok, d, chunk_frames, overlap_frames, sets)
    ws = alloc_workspace(nb, q.device) if workspace is None else workspace
    _check(lib().rehyat_forward_mlp(_p(q), _p(k), _p(v), _p(Wq1), _p(bq1), _p(Wq2), _p(bq2), _p(Wk1), _p(bk1),
                                    _p(Wk2), _p(bk2), B, H, F, S_tok, d, chunk_frames, overlap_frames, SETS[sets],
                                    LAYOUTS[layout], _p(out), _p(ws), ws.numel(), _stream()), "rehyat_forward_mlp")
    return out


def forward_host_workspace_bytes(B, H, F, S_tok, d, chunk_frames, overlap_frames, sets="causal") -> int:
    n = _c_size(0)
    _check(lib().rehyat_forward_host_workspace_bytes(B, H, F, S_tok, d, chunk_frames, overlap_frames, SETS[sets],
                                                     ctypes.byref(n)), "rehyat_forward_host_workspace_bytes")
    return n.value


def forward_host(q, k, v, F, S_tok, chunk_frames, overlap_frames, out, workspace, sets="causal", layout="bhnd",
                 stream=None):
    """rehyat_forward_host: q, k, v and out are HOST tensors (page-locked for
    asynchronous copies); workspace is a device uint8 tensor of
    forward_host_workspace_bytes(...) bytes.  Enqueued on `stream` (default:
    torch's current stream); synchronise before reading out."""
    for n_, t in (("q", q), ("k", k), ("v", v), ("out", out)):
        if not isinstance(t, torch.Tensor) or t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError(f"{n_} must be a contiguous bf16 host tensor")
    B, H, N, d = _dims(q, F, S_tok, layout)
    st = _vp(stream.cuda_stream) if stream is not None else _stream()
    _check(lib().rehyat_forward_host(_p(q), _p(k), _p(v), B, H, F, S_tok, d, chunk_frames, overlap_frames, SETS[sets],
                                     LAYOUTS[layout], _p(out), _p(workspace), workspace.numel(), st),
           "rehyat_forward_host")
    return out


def forward_capi(q, k, v, F, S_tok, chunk_frames, overlap_frames, out=None):
    """Same as forward() through rehyat_forward (library-allocated scratch)."""
    B, H, N, d = _shape(q, F, S_tok)
    out = torch.empty_like(q) if out is None else out
    _check(lib().rehyat_forward(_p(q), _p(k), _p(v), B, H, F, S_tok, d, chunk_frames, overlap_frames, _p(out),
                                _stream()), "rehyat_forward")
    return out


NOALLOC_SCRATCH_BYTES = 32 << 20


def forward_noalloc(q, k, v, F, S_tok, chunk_frames, overlap_frames, out):
    """rehyat_forward_noalloc: the forward with no device allocation at all
    (scratch in a fixed array inside the library; ``out`` must be given).
    For callers that cannot allocate during a call; calls on one device must
    not overlap on the GPU (they share the array)."""
    for n, t in (("q", q), ("k", k), ("v", v), ("out", out)):
        _need(t, torch.bfloat16, n)
    B, H, N, d = _shape(q, F, S_tok)
    _check(lib().rehyat_forward_noalloc(_p(q), _p(k), _p(v), B, H, F, S_tok, d, chunk_frames, overlap_frames,
                                        _p(out), _stream()), "rehyat_forward_noalloc")
    return out


def forward_states(k, v, F, S_tok, chunk_frames, overlap_frames, workspace):
    B, H, N, d = _shape(k, F, S_tok)
    _check(lib().rehyat_forward_states(_p(k), _p(v), B, H, F, S_tok, d, chunk_frames, overlap_frames, _p(workspace),
                                       workspace.numel(), _stream()), "rehyat_forward_states")


def forward_attention(q, k, v, F, S_tok, chunk_frames, overlap_frames, out, workspace):
    B, H, N, d = _shape(q, F, S_tok)
    _check(lib().rehyat_forward_attention(_p(q), _p(k), _p(v), B, H, F, S_tok, d, chunk_frames, overlap_frames,
                                          _p(out), _p(workspace), workspace.numel(), _stream()),
           "rehyat_forward_attention")


def forward_f32(q, k, v, F, S_tok, chunk_frames, overlap_frames, out=None):
    for n, t in (("q", q), ("k", k), ("v", v)):
        _need(t, torch.float32, n)
    B, H, N, d = _shape(q, F, S_tok)
    out = torch.empty_like(q) if out is None else out
    _check(lib().rehyat_forward_f32(_p(q), _p(k), _p(v), B, H, F, S_tok, d, chunk_frames, overlap_frames, _p(out),
                                    _stream()), "rehyat_forward_f32")
    return out


def forward_parts(q, k, v, F, S_tok, chunk_frames, overlap_frames):
    """Unnormalised terms of the joint normaliser: (aS, nS, aL, nL, M), fp32."""
    for n, t in (("q", q), ("k", k), ("v", v)):
        _need(t, torch.bfloat16, n)
    B, H, N, d = _shape(q, F, S_tok)
    f = dict(dtype=torch.float32, device=q.device)
    aS, aL = torch.empty(B, H, N, d, **f), torch.empty(B, H, N, d, **f)
    nS, nL, M = torch.empty(B, H, N, **f), torch.empty(B, H, N, **f), torch.empty(B, H, N, **f)
    _check(lib().rehyat_forward_parts(_p(q), _p(k), _p(v), B, H, F, S_tok, d, chunk_frames, overlap_frames, _p(aS),
                                      _p(nS), _p(aL), _p(nL), _p(M), _stream()), "rehyat_forward_parts")
    return aS, nS, aL, nL, M


def chunk_states(k, v, F, S_tok, chunk_frames, overlap_frames):
    """States entering each chunk: S [B,H,nc,2d,d], z [B,H,nc,2d] (fp32)."""
    for n, t in (("k", k), ("v", v)):
        _need(t, torch.bfloat16, n)
    B, H, N, d = _shape(k, F, S_tok)
    tc = min(chunk_frames, F)
    nc = -(-F // tc)
    S = torch.empty(B, H, nc, 2 * d, d, dtype=torch.float32, device=k.device)
    z = torch.empty(B, H, nc, 2 * d, dtype=torch.float32, device=k.device)
    _check(lib().rehyat_chunk_states(_p(k), _p(v), B, H, F, S_tok, d, chunk_frames, overlap_frames, _p(S), _p(z),
                                     _stream()), "rehyat_chunk_states")
    return S, z


# --------------------------------------------------------------------------- #
# recurrent form                                                               #
# --------------------------------------------------------------------------- #
def step_workspace_bytes(B, H, S_tok, d, q_frames, ctx_frames, evict_frames) -> int:
    n = _c_size(0)
    _check(lib().rehyat_step_workspace_bytes(B, H, S_tok, d, q_frames, ctx_frames, evict_frames, ctypes.byref(n)),
           "rehyat_step_workspace_bytes")
    return n.value


def step(q_c, k_c, v_c, state_S, state_z, S_tok, q_frames, ctx_frames, evict_frames, out=None, workspace=None,
         capi=False):
    """One chunk of the recurrent form (bf16); state_S/state_z updated in place."""
    for n, t in (("q_c", q_c), ("k_c", k_c), ("v_c", v_c)):
        _need(t, torch.bfloat16, n)
    _need(state_S, torch.float32, "state_S")
    _need(state_z, torch.float32, "state_z", 3)
    B, H, Lq, d = q_c.shape
    if Lq != q_frames * S_tok or k_c.shape[2] != (ctx_frames + q_frames) * S_tok:
        raise ValueError("q_c / k_c lengths do not match the frame counts")
    out = torch.empty_like(q_c) if out is None else out
    if capi:
        _check(lib().rehyat_step(_p(q_c), _p(k_c), _p(v_c), _p(state_S), _p(state_z), _p(out), B, H, S_tok, d,
                                 q_frames, ctx_frames, evict_frames, _stream()), "rehyat_step")
        return out
    nb = step_workspace_bytes(B, H, S_tok, d, q_frames, ctx_frames, evict_frames)
    ws = alloc_workspace(nb, q_c.device) if workspace is None else workspace
    _check(lib().rehyat_step_ws(_p(q_c), _p(k_c), _p(v_c), _p(state_S), _p(state_z), _p(out), B, H, S_tok, d,
                                q_frames, ctx_frames, evict_frames, _p(ws), ws.numel(), _stream()), "rehyat_step_ws")
    return out


def step_ex(q_c, k_c, v_c, state_S, state_z, S_tok, q_frames, ctx_frames, evict_frames, layout="bhnd", out=None,
            workspace=None):
    """rehyat_step_ex: one chunk of the recurrent form on [B,H,L,d] ("bhnd")
    or [B,L,H,d] ("bnhd") tensors."""
    for n, t in (("q_c", q_c), ("k_c", k_c), ("v_c", v_c)):
        _need(t, torch.bfloat16, n)
    _need(state_S, torch.float32, "state_S")
    _need(state_z, torch.float32, "state_z", 3)
    if layout == "bhnd":
        B, H, Lq, d = q_c.shape
        Lk = k_c.shape[2]
    else:
        B, Lq, H, d = q_c.shape
        Lk = k_c.shape[1]
    if Lq != q_frames * S_tok or Lk != (ctx_frames + q_frames) * S_tok:
        raise ValueError("q_c / k_c lengths do not match the frame counts")
    out = torch.empty_like(q_c) if out is None else out
    ws = workspace
    _check(lib().rehyat_step_ex(_p(q_c), _p(k_c), _p(v_c), _p(state_S), _p(state_z), _p(out), B, H, S_tok, d,
                                q_frames, ctx_frames, evict_frames, LAYOUTS[layout], _p(ws),
                                ws.numel() if ws is not None else 0, _stream()), "rehyat_step_ex")
    return out


def step_phi(q_c, k_c, v_c, phi_q_c, phi_k_c, state_S, state_z, S_tok, q_frames, ctx_frames, evict_frames,
             out=None, workspace=None):
    """rehyat_step_phi: one chunk of the recurrent form with precomputed
    features phi_q_c [B,H,Lq,2d] and phi_k_c [B,H,Lk,2d] (bf16)."""
    for n, t in (("q_c", q_c), ("k_c", k_c), ("v_c", v_c), ("phi_q_c", phi_q_c), ("phi_k_c", phi_k_c)):
        _need(t, torch.bfloat16, n)
    _need(state_S, torch.float32, "state_S")
    _need(state_z, torch.float32, "state_z", 3)
    B, H, Lq, d = q_c.shape
    if Lq != q_frames * S_tok or k_c.shape[2] != (ctx_frames + q_frames) * S_tok:
        raise ValueError("q_c / k_c lengths do not match the frame counts")
    if tuple(phi_q_c.shape) != (B, H, Lq, 2 * d) or tuple(phi_k_c.shape) != (B, H, k_c.shape[2], 2 * d):
        raise ValueError("phi_q_c / phi_k_c must be [B, H, L, 2d] for the chunk's queries / window keys")
    out = torch.empty_like(q_c) if out is None else out
    ws = workspace
    _check(lib().rehyat_step_phi(_p(q_c), _p(k_c), _p(v_c), _p(phi_q_c), _p(phi_k_c), _p(state_S), _p(state_z),
                                 _p(out), B, H, S_tok, d, q_frames, ctx_frames, evict_frames, _p(ws),
                                 ws.numel() if ws is not None else 0, _stream()), "rehyat_step_phi")
    return out


def phi_mlp_f32(x, W1, b1, W2, b2, out=None):
    """rehyat_phi_mlp_f32: the learned feature map in fp32, x [B,H,N,d]
    float, weights float -> phi [B,H,N,2d] float."""
    _need(x, torch.float32, "x")
    B, H, N, d = x.shape
    for n, t, shape in (("W1", W1, (H, 2 * d, d)), ("b1", b1, (H, 2 * d)), ("W2", W2, (H, 2 * d, 2 * d)),
                        ("b2", b2, (H, 2 * d))):
        _need(t, torch.float32, n, len(shape))
        if tuple(t.shape) != shape:
            raise ValueError(f"{n} must be {shape}")
    out = torch.empty((B, H, N, 2 * d), dtype=torch.float32, device=x.device) if out is None else out
    _check(lib().rehyat_phi_mlp_f32(_p(x), B, H, N, d, _p(W1), _p(b1), _p(W2), _p(b2), _p(out), _stream()),
           "rehyat_phi_mlp_f32")
    return out


def forward_phi_f32(q, k, v, phi_q, phi_k, F, S_tok, chunk_frames, overlap_frames, out=None):
    """rehyat_forward_phi_f32: the fp32 forward with precomputed features."""
    for n, t in (("q", q), ("k", k), ("v", v), ("phi_q", phi_q), ("phi_k", phi_k)):
        _need(t, torch.float32, n)
    B, H, N, d = _shape(q, F, S_tok)
    out = torch.empty_like(q) if out is None else out
    _check(lib().rehyat_forward_phi_f32(_p(q), _p(k), _p(v), _p(phi_q), _p(phi_k), B, H, F, S_tok, d, chunk_frames,
                                        overlap_frames, _p(out), _stream()), "rehyat_forward_phi_f32")
    return out


def step_f32(q_c, k_c, v_c, state_S, state_z, S_tok, q_frames, ctx_frames, evict_frames, out=None):
    for n, t in (("q_c", q_c), ("k_c", k_c), ("v_c", v_c)):
        _need(t, torch.float32, n)
    B, H, Lq, d = q_c.shape
    out = torch.empty_like(q_c) if out is None else out
    _check(lib().rehyat_step_f32(_p(q_c), _p(k_c), _p(v_c), _p(state_S), _p(state_z), _p(out), B, H, S_tok, d,
                                 q_frames, ctx_frames, evict_frames, _stream()), "rehyat_step_f32")
    return out


def step_frames(t: int, F: int, chunk_frames: int, overlap_frames: int):
    """(q0_frame, w_t, ctx_frames, q_frames, evict_frames) for chunk t of a
    video streamed through step(): window start w_t = max(t*T_c - T_o, 0)."""
    tc = min(chunk_frames, F)
    to = min(overlap_frames, F)
    f0 = t * tc
    w = max(f0 - to, 0)
    qf = min(tc, F - f0)
    end = f0 + qf
    w_next = min(max((t + 1) * tc - to, 0), end)
    return f0, w, f0 - w, qf, w_next - w


# --------------------------------------------------------------------------- #
# feature map, status                                                          #
# --------------------------------------------------------------------------- #
def phi(x: torch.Tensor, out_dtype=None) -> torch.Tensor:
    if x.dtype not in (torch.bfloat16, torch.float32) or not x.is_cuda or not x.is_contiguous():
        raise ValueError("x must be a contiguous CUDA bf16/f32 tensor")
    od = out_dtype or x.dtype
    d = x.shape[-1]
    rows = x.numel() // d
    y = torch.empty(*x.shape[:-1], 2 * d, dtype=od, device=x.device)
    code = lambda dt: DTYPE_BF16 if dt == torch.bfloat16 else DTYPE_F32
    _check(lib().rehyat_phi(_p(x), code(x.dtype), _p(y), code(od), rows, d, _stream()), "rehyat_phi")
    return y


def wait_probe(gave_up=None):
    """rehyat_wait_probe: one warp waits on a barrier nothing completes; the
    bounded wait gives up after its limit.  gave_up: optional int32 device
    tensor of one element, set to 1 when the wait gave up."""
    if gave_up is not None:
        _need(gave_up, torch.int32, "gave_up", 1)
    _check(lib().rehyat_wait_probe(_p(gave_up), _stream()), "rehyat_wait_probe")


def device_status() -> int:
    """Status of device-side bounded waits since the last query (synchronises)."""
    detail = ctypes.c_uint(0)
    return lib().rehyat_device_status(ctypes.byref(detail))
