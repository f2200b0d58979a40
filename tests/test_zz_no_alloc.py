"""The no-allocation entry point: rehyat_hybrid_attn_fwd_noalloc.

Some callers cannot allocate device memory (code running under another
runtime's allocator or memory pool, plug-in hosts that forbid allocation
after start-up, tools that only pass along buffers they were given), so they
cannot supply the workspace rehyat_hybrid_attn_fwd needs.  The no-alloc
variant takes its scratch from a fixed 32 MiB array inside the library.

This file runs last (pytest collects it last by name), so a failure here
never hides the results of the other tests.  It must pass alone in a fresh
process and after the others: it does not depend on any earlier call having
looked up the scratch address.
"""
import numpy as np
import pytest
import torch

import linear_attention_video_chunked_b200 as rh
from rehyat_inputs import make_problem
from tests.gpu_util import device_tensors, err_stats

pytestmark = pytest.mark.gpu


def _params(p):
    return rh.make_params(batch=p.batch, heads=p.heads, T=p.T, Hs=p.Hs, Ws=p.Ws, D=p.D, Dp=p.Dp,
                          Tc=p.Tc, To=p.To, causal=p.causal, in_dtype=rh.BF16, out_dtype=rh.F32)


def _with_workspace(p, dev):
    """The regular entry point, with a caller-allocated workspace."""
    return rh.hybrid_attn(dev["q"], dev["k"], dev["v"], dev["Wq"], dev["bq"], dev["Wk"], dev["bk"],
                          T=p.T, Hs=p.Hs, Ws=p.Ws, Tc=p.Tc, To=p.To, causal=p.causal)


def _no_alloc(p, dev):
    """The no-alloc entry point through the C ABI: inputs and output only."""
    y = torch.empty(p.batch, p.heads, p.N, p.D, device="cuda", dtype=torch.float32)
    phi = rh.RehyatPhi(dev["Wq"].data_ptr(), dev["bq"].data_ptr(), dev["Wk"].data_ptr(),
                       dev["bk"].data_ptr())
    st = rh.rehyat_hybrid_attn_fwd_noalloc(_params(p), dev["q"].data_ptr(), dev["k"].data_ptr(),
                                           dev["v"].data_ptr(), phi, y.data_ptr(), None,
                                           torch.cuda.current_stream().cuda_stream)
    assert st == 0, rh.rehyat_status_string(st)
    return y


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    rh.lib()


def test_no_alloc_matches_workspace_entry_point_two_calls_in_a_row():
    # Two different problems back to back: the second call reuses the
    # scratch the first one left behind.
    problems = [
        make_problem(batch=1, heads=4, T=9, Hs=12, Ws=20, D=128, Dp=128, Tc=3, To=1,
                     causal=False, dtype="bf16", seed=71),
        make_problem(batch=1, heads=3, T=7, Hs=10, Ws=13, D=128, Dp=64, Tc=2, To=2,
                     causal=True, dtype="bf16", seed=72),
    ]
    # Both entry points run the same deterministic kernels on the same
    # inputs, so the outputs must be bit-identical: a scratch region that one
    # call failed to overwrite would show up here even if its effect were
    # small.
    for p in problems:
        dev = device_tensors(p)
        y_ref = _with_workspace(p, dev)
        y = _no_alloc(p, dev)
        torch.cuda.synchronize()
        assert torch.equal(y, y_ref), err_stats(y.double().cpu().numpy(),
                                                y_ref.double().cpu().numpy())
        assert np.isfinite(y.cpu().numpy()).all()


def test_no_alloc_refuses_problems_over_its_scratch():
    # One batch-2 21x30x52 layer with 12 heads needs ~45 MiB of workspace.
    p = rh.make_params(batch=2, heads=12, T=21, Hs=30, Ws=52, D=128, Dp=128, Tc=3, To=1,
                       causal=0, in_dtype=rh.BF16, out_dtype=rh.F32)
    assert rh.rehyat_workspace_bytes(p) > 32 << 20
    phi = rh.RehyatPhi(4096, 4096, 4096, 4096)
    st = rh.rehyat_hybrid_attn_fwd_noalloc(p, 4096, 4096, 4096, phi, 4096, None, None)
    assert st == 6 and rh.STATUS[st] == "REHYAT_ERR_SCRATCH_LIMIT"
