"""C ABI checks that need no GPU: the library loads, exports every entry point
declared in include/rehyat.h, and validates arguments on the host (returning a
status without touching CUDA)."""
import ctypes
import os
import re

import pytest

from linear_attention_video_chunk_b200 import build as rbuild
from linear_attention_video_chunk_b200 import rehyat as R

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "rehyat.h")


@pytest.fixture(scope="module")
def lib():
    rbuild.build()
    return R.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(rehyat_\w+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("rehyat_forward", "rehyat_forward_f32", "rehyat_step", "rehyat_step_f32",
              "rehyat_forward_parts", "rehyat_status_string"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_covers_every_symbol():
    assert set(declared_functions()) <= set(R._SIGS)


def test_only_c_abi_symbols_are_exported(lib):
    out = os.popen(f"nm -D --defined-only {R.LIB_PATH}").read()
    syms = [l.split()[-1] for l in out.splitlines() if " T " in l]
    assert syms and all(s.startswith("rehyat_") for s in syms), syms


def test_status_strings(lib):
    for st in range(6):
        assert R.status_string(st).startswith("REHYAT_")
    assert "UNKNOWN" in R.status_string(99)


def _fwd(lib, q=16, k=16, v=16, out=16, B=1, H=1, F=4, S=8, d=64, Tc=2, To=1):
    return lib.rehyat_forward(q, k, v, B, H, F, S, d, Tc, To, out, None)


def test_forward_validation(lib):
    assert _fwd(lib, q=0) == R.EINVAL                     # null pointer
    assert _fwd(lib, k=8) == R.EINVAL                     # 16-byte misaligned
    assert _fwd(lib, d=96) == R.EUNSUPPORTED
    assert _fwd(lib, d=0) == R.EINVAL
    assert _fwd(lib, F=0) == R.EINVAL
    assert _fwd(lib, S=0) == R.EINVAL
    assert _fwd(lib, Tc=0) == R.EINVAL
    assert _fwd(lib, To=-1) == R.EINVAL
    assert _fwd(lib, B=-1) == R.EINVAL
    assert _fwd(lib, F=1 << 20, S=1 << 12) == R.EINVAL   # N overflows int
    assert lib.rehyat_forward_f32(0, 16, 16, 1, 1, 4, 8, 64, 2, 1, 16, None) == R.EINVAL
    assert lib.rehyat_forward_parts(16, 16, 16, 1, 1, 4, 8, 64, 2, 1, 0, 16, 16, 16, 16, None) == R.EINVAL


def test_step_validation(lib):
    st = lambda **kw: lib.rehyat_step(*(kw.get(n, 16) for n in ("q", "k", "v", "S", "z", "o")),
                                      1, 1, 8, kw.get("d", 64), kw.get("qf", 2), kw.get("cf", 1),
                                      kw.get("ef", 1), None)
    assert st(S=0) == R.EINVAL
    assert st(z=4) == R.EINVAL
    assert st(ef=4) == R.EINVAL        # evict beyond the window
    assert st(qf=0) == R.EINVAL
    assert st(cf=-1) == R.EINVAL
    assert st(d=32) == R.EUNSUPPORTED


def test_chunk_states_validation(lib):
    # k, v, S: 16-byte aligned device pointers; z: non-null
    f = lib.rehyat_chunk_states
    assert f(16, 16, 1, 1, 4, 8, 64, 2, 1, 0, 16, None) == R.EINVAL    # null S
    assert f(16, 16, 1, 1, 4, 8, 64, 2, 1, 20, 16, None) == R.EINVAL   # S at 4 mod 16
    assert f(16, 16, 1, 1, 4, 8, 64, 2, 1, 16, 0, None) == R.EINVAL    # null z
    assert f(8, 16, 1, 1, 4, 8, 64, 2, 1, 16, 16, None) == R.EINVAL    # misaligned k


def test_workspace_sizes(lib):
    a = R.workspace_bytes(1, 12, 21, 1560, 128, 3, 1)
    b = R.workspace_bytes(1, 12, 41, 1560, 128, 3, 1)
    assert 0 < a < b and a % 256 == 0
    # the states of 7 chunks (bf16 hi + lo + fp32 z) are part of it
    assert a >= 12 * 7 * 256 * 128 * 2 * 2
    assert R.workspace_bytes(1, 1, 4, 8, 64, 4, 0) >= 256          # one chunk: no segments
    assert R.step_workspace_bytes(1, 12, 1560, 128, 3, 1, 3) > 0
    n = ctypes.c_size_t(0)
    assert lib.rehyat_forward_workspace_bytes(1, 1, 4, 8, 64, 2, 1, None) == R.EINVAL
    assert lib.rehyat_forward_workspace_bytes(1, 1, 4, 8, 100, 2, 1, ctypes.byref(n)) == R.EUNSUPPORTED


def test_ws_variants_check_workspace(lib):
    # workspace too small -> ENOMEM before any launch; misaligned -> EINVAL
    assert lib.rehyat_forward_ws(16, 16, 16, 1, 1, 4, 8, 64, 2, 1, 16, 256, 1, None) == R.ENOMEM
    assert lib.rehyat_forward_ws(16, 16, 16, 1, 1, 4, 8, 64, 2, 1, 16, 272, 1 << 30, None) == R.EINVAL


def test_forward_ex_validation(lib):
    f = lambda sets, ws=0, nb=0, layout=0: lib.rehyat_forward_ex(16, 16, 16, 1, 1, 4, 8, 64, 2, 1, sets, layout,
                                                                   16, ws, nb, None)
    assert f(2) == R.EINVAL              # unknown set mode
    assert f(0, layout=2) == R.EINVAL    # unknown layout
    assert f(-1) == R.EINVAL
    assert f(1, ws=256, nb=1) == R.ENOMEM  # workspace too small (checked before launching)
    assert f(1, ws=272, nb=1 << 30) == R.EINVAL  # misaligned workspace
    n0, n1 = ctypes.c_size_t(0), ctypes.c_size_t(0)
    assert lib.rehyat_forward_ex_workspace_bytes(1, 12, 21, 1560, 128, 3, 1, 0, ctypes.byref(n0)) == R.OK
    assert lib.rehyat_forward_ex_workspace_bytes(1, 12, 21, 1560, 128, 3, 1, 1, ctypes.byref(n1)) == R.OK
    assert n0.value == R.workspace_bytes(1, 12, 21, 1560, 128, 3, 1) and n1.value > 0


def test_phi_validation(lib):
    assert lib.rehyat_phi(0, 0, 16, 0, 4, 64, None) == R.EINVAL
    assert lib.rehyat_phi(16, 3, 16, 0, 4, 64, None) == R.EINVAL
    assert lib.rehyat_phi(16, 0, 16, 0, 0, 64, None) == R.EINVAL


def test_step_frames_cover_the_video():
    """Host logic of the streaming driver: windows and evictions tile [0, F)."""
    for F, Tc, To in [(21, 3, 1), (81, 3, 1), (7, 2, 3), (10, 4, 0), (5, 7, 2)]:
        folded = 0
        t = 0
        while t * min(Tc, F) < F:
            f0, w, cf, qf, ef = R.step_frames(t, F, Tc, To)
            assert w == folded and cf == f0 - w and qf >= 1
            folded += ef
            t += 1
        assert folded <= F


def test_mlp_validation(lib):
    def m(**kw):
        a = dict(x=16, N=100, d=128, layout=0, W1=16, b1=16, W2=16, b2=16, phi=16)
        a.update(kw)
        return lib.rehyat_phi_mlp(a["x"], 1, 2, a["N"], a["d"], a["layout"], a["W1"], a["b1"], a["W2"], a["b2"],
                                  a["phi"], None)
    assert m(x=0) == R.EINVAL
    assert m(W2=8) == R.EINVAL           # misaligned weights
    assert m(b1=0) == R.EINVAL
    assert m(phi=0) == R.EINVAL
    assert m(d=96) == R.EUNSUPPORTED
    assert m(N=0) == R.EINVAL
    assert m(layout=3) == R.EINVAL

    def fp(phi_q=16, phi_k=16, sets=0, ws=0, nb=0):
        return lib.rehyat_forward_phi(16, 16, 16, phi_q, phi_k, 1, 1, 4, 8, 64, 2, 1, sets, 0, 16, ws, nb, None)
    assert fp(phi_q=0) == R.EINVAL
    assert fp(phi_k=24) == R.EINVAL
    assert fp(sets=2) == R.EINVAL
    assert fp(ws=256, nb=1) == R.ENOMEM

    def fm(wk2=16, ws=0, nb=0, d=64):
        return lib.rehyat_forward_mlp(16, 16, 16, 16, 16, 16, 16, 16, 16, wk2, 16, 1, 1, 4, 8, d, 2, 1, 0, 0, 16,
                                      ws, nb, None)
    assert fm(wk2=0) == R.EINVAL
    assert fm(d=32) == R.EUNSUPPORTED
    assert fm(ws=256, nb=1) == R.ENOMEM


def test_mlp_workspace_holds_both_feature_maps():
    ex = ctypes.c_size_t(0)
    R.lib().rehyat_forward_ex_workspace_bytes(1, 12, 21, 1560, 128, 3, 1, 0, ctypes.byref(ex))
    phi = 12 * 21 * 1560 * 256 * 2            # [B, H, N, 2d] bf16, a multiple of 256 here
    assert R.forward_mlp_workspace_bytes(1, 12, 21, 1560, 128, 3, 1) == ex.value + 2 * phi


def test_step_phi_validation(lib):
    def sp(**kw):
        a = dict(q=16, pq=16, pk=16, S=16, ef=1, ws=0, nb=0)
        a.update(kw)
        return lib.rehyat_step_phi(a["q"], 16, 16, a["pq"], a["pk"], a["S"], 16, 16, 1, 1, 8, 64, 2, 1, a["ef"],
                                   a["ws"], a["nb"], None)
    assert sp(pq=0) == R.EINVAL
    assert sp(pk=8) == R.EINVAL
    assert sp(S=0) == R.EINVAL
    assert sp(ef=4) == R.EINVAL          # evict beyond the window
    assert sp(ws=256, nb=1) == R.ENOMEM


def test_forward_host_validation(lib):
    def fh(q=16, ws=256, nb=1 << 40, d=64):
        return lib.rehyat_forward_host(q, 16, 16, 1, 1, 4, 8, d, 2, 1, 0, 0, 16, ws, nb, None)
    assert fh(q=0) == R.EINVAL
    assert fh(ws=0) == R.EINVAL
    assert fh(ws=272) == R.EINVAL        # misaligned workspace
    assert fh(nb=1) == R.ENOMEM
    assert fh(d=96) == R.EUNSUPPORTED
    ex = ctypes.c_size_t(0)
    lib.rehyat_forward_ex_workspace_bytes(1, 12, 21, 1560, 128, 3, 1, 0, ctypes.byref(ex))
    assert R.forward_host_workspace_bytes(1, 12, 21, 1560, 128, 3, 1) == ex.value + 4 * 12 * 32760 * 128 * 2


def test_f32_learned_phi_validation(lib):
    assert lib.rehyat_phi_mlp_f32(0, 1, 1, 8, 64, 16, 16, 16, 16, 16, None) == R.EINVAL
    assert lib.rehyat_phi_mlp_f32(16, 1, 1, 8, 96, 16, 16, 16, 16, 16, None) == R.EUNSUPPORTED
    assert lib.rehyat_phi_mlp_f32(16, 1, 1, 0, 64, 16, 16, 16, 16, 16, None) == R.EINVAL
    assert lib.rehyat_forward_phi_f32(16, 16, 16, 0, 16, 1, 1, 4, 8, 64, 2, 1, 16, None) == R.EINVAL
    assert lib.rehyat_forward_phi_f32(16, 16, 16, 16, 24, 1, 1, 4, 8, 64, 2, 1, 16, None) == R.EINVAL


def test_step_ex_validation(lib):
    def se(layout=0, ws=0, nb=0, q=16):
        return lib.rehyat_step_ex(q, 16, 16, 16, 16, 16, 1, 1, 8, 64, 2, 1, 1, layout, ws, nb, None)
    assert se(layout=2) == R.EINVAL
    assert se(q=0) == R.EINVAL
    assert se(ws=256, nb=1) == R.ENOMEM
    assert se(ws=272, nb=1 << 30) == R.EINVAL


def _header_signatures():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    out = {}
    for ret, name, args in re.findall(r"\b([\w ]+?\*?)\s*\b(rehyat_\w+)\s*\(([^)]*)\)\s*;", src):
        a = args.strip()
        out[name] = (ret.strip(), [] if a in ("", "void") else [x.strip() for x in a.split(",")])
    return out


def _ctype_of(decl):
    """Coarse ctypes class of one C parameter declaration."""
    if "*" in decl:
        return "ptr"
    t = decl.rsplit(" ", 1)[0].strip()
    return {"int": "int", "int64_t": "int64", "size_t": "size_t", "float": "float"}[t]


def test_binding_argtypes_match_the_header():
    """Every binding's ctypes argument list has the header's arity and, per
    position, the same kind (pointer / int / int64 / size_t), so no call marshals
    an argument into the wrong slot."""
    kind = {ctypes.c_void_p: "ptr", ctypes.c_int: "int", ctypes.c_int64: "int64", ctypes.c_size_t: "size_t",
            ctypes.c_float: "float"}
    sigs = _header_signatures()
    assert len(sigs) == len(declared_functions())
    for name, (ret, params) in sigs.items():
        want = [_ctype_of(p) for p in params]
        got = [kind.get(t, "ptr") for t in R._SIGS[name]]
        assert got == want, (name, got, want)
        assert (R._RESTYPES.get(name, ctypes.c_int) is ctypes.c_char_p) == ret.startswith("const char")


def _undocumented(lines):
    """Declarations with no comment block closing right above them or above
    the contiguous group of declaration / #define lines they belong to."""
    out = []
    for i, l in enumerate(lines):
        m = re.match(r"^\s*(?:const\s+)?\w[\w\s*]*?\b(rehyat_\w+)\s*\(", l)
        if not m or l.lstrip().startswith(("*", "/*")):
            continue
        j = i - 1
        while j >= 0 and lines[j].strip() and not lines[j].strip().endswith("*/"):
            j -= 1
        if j < 0 or not lines[j].strip().endswith("*/"):
            out.append(m.group(1))
    return out


def test_every_declaration_is_documented():
    """Each entry point in the header has a comment block right above it, or
    belongs to a group of declarations (or a #define) that the block right
    above the group documents."""
    lines = open(HEADER).read().splitlines()
    assert not _undocumented(lines), _undocumented(lines)
    # the check itself catches a declaration whose comment is removed
    k = next(i for i, l in enumerate(lines) if l.startswith("int rehyat_step_ex("))
    j = k - 1
    while not lines[j].lstrip().startswith("/*"):
        j -= 1
    assert "rehyat_step_ex" in _undocumented(lines[:j] + [""] + lines[k:])


# Pointer arguments that may be NULL by contract (besides `stream`): the
# workspace of the calls that then allocate stream-ordered scratch.
_NULLABLE = {(n, "workspace") for n in ("rehyat_forward_ex", "rehyat_forward_phi", "rehyat_forward_mlp",
                                         "rehyat_step_ex", "rehyat_step_phi")}
_SIZES = dict(B=1, H=1, F=4, S_tok=8, N=32, d=64, chunk_frames=2, overlap_frames=1, sets=0, layout=0, q_frames=2,
              ctx_frames=1, evict_frames=1, x_dtype=0, y_dtype=0, rows=4, n=4, workspace_bytes=1 << 30)


@pytest.mark.skipif(__import__("torch").cuda.is_available(),
                    reason="passes fake device addresses; host-only check")
def test_each_required_pointer_is_validated(lib):
    """For every entry point and every required pointer argument: with valid
    sizes, that pointer NULL and every other pointer a fake aligned address,
    the call returns REHYAT_EINVAL before any CUDA call (a call that went on
    would fail in CUDA here, with no device, and return something else)."""
    size_out = ctypes.c_size_t(0)
    missing = []
    for name, (ret, params) in _header_signatures().items():
        if name in ("rehyat_wait_probe", "rehyat_device_status", "rehyat_status_string"):
            continue
        names = [p.replace("*", " ").split()[-1] for p in params]
        for k, p in enumerate(params):
            if "*" not in p or names[k] == "stream" or (name, names[k]) in _NULLABLE:
                continue
            vals = []
            for i, (q, pn) in enumerate(zip(params, names)):
                if "*" not in q:
                    vals.append(_SIZES[pn])
                elif i == k or pn == "stream":
                    vals.append(None)
                else:
                    vals.append(ctypes.byref(size_out) if pn == "bytes" else 0x10000)
            if getattr(lib, name)(*vals) != R.EINVAL:
                missing.append((name, names[k]))
    assert not missing, missing


def test_elementwise_calls_check_element_alignment(lib):
    assert lib.rehyat_phi(0x10001, 0, 0x10000, 0, 4, 64, None) == R.EINVAL       # bf16 x at an odd address
    assert lib.rehyat_phi(0x10000, 1, 0x10002, 1, 4, 64, None) == R.EINVAL       # fp32 y at 2 mod 4
    assert lib.rehyat_phi(0x10000, 2, 0x10000, 0, 4, 64, None) == R.EINVAL       # unknown dtype


_BAD_SIZES = dict(B=[0, -1], H=[0], F=[0], S_tok=[0], N=[0], d=[96, 0], chunk_frames=[0], overlap_frames=[-1],
                  sets=[2, -1], layout=[2, -1], q_frames=[0], ctx_frames=[-1], evict_frames=[-1, 4], x_dtype=[2],
                  y_dtype=[2], rows=[0], n=[0])


@pytest.mark.skipif(__import__("torch").cuda.is_available(),
                    reason="passes fake device addresses; host-only check")
def test_each_size_argument_is_validated(lib):
    """For every entry point and every size / mode argument: one invalid value
    (zero or negative counts, d outside {64, 128}, unknown set mode, layout
    or dtype, more evicted frames than the window holds), every other argument
    valid, returns REHYAT_EINVAL or REHYAT_EUNSUPPORTED before any CUDA call."""
    missing = []
    for name, (ret, params) in _header_signatures().items():
        if name in ("rehyat_wait_probe", "rehyat_device_status", "rehyat_status_string"):
            continue
        names = [p.replace("*", " ").split()[-1] for p in params]
        for k, pn in enumerate(names):
            if "*" in params[k] or pn == "workspace_bytes":
                continue
            for bad in _BAD_SIZES[pn]:
                if name == "rehyat_phi" and pn == "d" and bad > 0:
                    continue  # the element-wise map takes any d >= 1
                vals = []
                for i, (q, n2) in enumerate(zip(params, names)):
                    if "*" not in q:
                        vals.append(bad if i == k else _SIZES[n2])
                    elif n2 == "stream":
                        vals.append(None)
                    else:
                        vals.append(ctypes.byref(ctypes.c_size_t(0)) if n2 == "bytes" else 0x10000)
                if getattr(lib, name)(*vals) not in (R.EINVAL, R.EUNSUPPORTED):
                    missing.append((name, pn, bad))
    assert not missing, missing
