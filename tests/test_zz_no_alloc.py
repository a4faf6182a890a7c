"""rehyat_forward_noalloc: the forward for callers that cannot allocate.

Callers such as a server that reserves all device memory at start-up, or a
plugin whose framework owns the allocator, cannot let the library allocate
scratch during a call.  rehyat_forward_noalloc keeps its scratch in a fixed
array inside the library instead.  These checks call it through the C ABI
and compare it with rehyat_forward, the allocating entry point, on two calls
in a row with different inputs (the second call must not see stale scratch
from the first), and check that a problem too large for the array is
refused before anything is launched.
"""
import ctypes

import numpy as np
import pytest
import torch

from linear_attention_video_chunk_b200 import inputs
from linear_attention_video_chunk_b200 import rehyat as R

pytestmark = pytest.mark.gpu

BF16_L2, BF16_MAX = 1e-2, 3e-2   # the bf16 tolerance of the other parity tests


def _close(y, ref):
    """(rel L2, max-abs / RMS) of y against ref.  Both are bf16 outputs of
    the same computation whose fp32 sums ran in a different order (the array
    version merges key pieces), so an element may round to the neighbouring
    bf16 value: one bf16 ulp of |ref| is allowed before the max-abs term."""
    y = y.double().cpu().numpy()
    ref = ref.double().cpu().numpy()
    e2 = (np.sqrt(((y - ref) ** 2).sum((-2, -1))) / np.sqrt((ref ** 2).sum((-2, -1)))).max()
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref), 1e-30))) - 7)
    em = np.maximum(np.abs(y - ref) - ulp, 0).max() / np.sqrt((ref ** 2).mean())
    return e2, em


def test_noalloc_matches_forward_on_two_calls_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    # the Wan2.1-1.3B 480p shape: its default scratch layout (~30 MB) fits
    # the 32 MiB array as it is
    B, H, d, F, S, Tc, To = 1, 12, 128, 21, 1560, 3, 1
    L = R.lib()
    for seed in (1, 5):
        q, k, v = (x.cuda() for x in inputs.make_qkv(B, H, F * S, d, seed, rms_qk=True))
        ref = R.forward_capi(q, k, v, F, S, Tc, To)
        out = torch.full_like(q, float("nan"))
        st = L.rehyat_forward_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), B, H, F, S, d, Tc, To,
                                      out.data_ptr(), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == R.OK, R.status_string(st)
        torch.cuda.synchronize()
        assert torch.isfinite(out.float()).all()
        e2, em = _close(out, ref)
        assert e2 <= BF16_L2 and em <= BF16_MAX, (seed, e2, em)
        if R.workspace_bytes(B, H, F, S, d, Tc, To) <= R.NOALLOC_SCRATCH_BYTES:
            # same scratch layout as rehyat_forward: same kernels, same order
            assert torch.equal(out, ref)
    assert R.device_status() == R.OK


def test_noalloc_merges_key_pieces_when_the_default_layout_does_not_fit():
    """B=1, H=37, d=128, F=9 x 64 tokens, T_c=3, T_o=1: the default layout
    sums each key segment in two pieces (~34 MB of scratch, more than the
    array); the array version sums them in one piece (~24 MB), so its result
    differs from rehyat_forward's only by fp32 summation order."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    B, H, d, F, S, Tc, To = 1, 37, 128, 9, 64, 3, 1
    assert R.workspace_bytes(B, H, F, S, d, Tc, To) > R.NOALLOC_SCRATCH_BYTES
    L = R.lib()
    for seed in (6, 7):
        q, k, v = (x.cuda() for x in inputs.make_qkv(B, H, F * S, d, seed, rms_qk=True))
        ref = R.forward_capi(q, k, v, F, S, Tc, To)
        out = torch.full_like(q, float("nan"))
        st = L.rehyat_forward_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), B, H, F, S, d, Tc, To,
                                      out.data_ptr(), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == R.OK, R.status_string(st)
        torch.cuda.synchronize()
        assert torch.isfinite(out.float()).all()
        e2, em = _close(out, ref)
        assert e2 <= BF16_L2 and em <= BF16_MAX, (seed, e2, em)
    assert R.device_status() == R.OK


def test_noalloc_refuses_a_problem_larger_than_its_array():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    # H = 64 at the 1.3B frame shape needs ~59 MB of chunk states alone:
    # refused with REHYAT_ENOMEM before any launch (the small buffers are
    # never touched)
    buf = torch.empty(4096, dtype=torch.bfloat16, device="cuda")
    p = buf.data_ptr()
    st = R.lib().rehyat_forward_noalloc(p, p, p, 1, 64, 21, 1560, 128, 3, 1, p, None)
    assert st == R.ENOMEM
    assert "ENOMEM" in R.status_string(st)
