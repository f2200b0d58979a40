"""GPU tests of the host-buffer forward (rehyat_hybrid_attn_fwd_host): slabs
of heads uploaded, computed and downloaded on three streams give exactly the
device forward's y (the per-(b,h) kernels do the same arithmetic whatever
the slab), for ragged head groups, slot reuse, pinned and pageable memory,
and both forms; a short workspace is refused."""
import pytest
import torch

import linear_attention_video_chunked_b200 as rh
from rehyat_inputs import make_problem
from tests.gpu_util import device_tensors

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    rh.lib()
    rh.rehyat_device_error_flags(reset=True)
    yield
    assert rh.rehyat_device_error_flags() == 0


def _device_y(p, dev):
    y = rh.hybrid_attn(dev["q"], dev["k"], dev["v"], dev["Wq"], dev["bq"], dev["Wk"], dev["bk"],
                       T=p.T, Hs=p.Hs, Ws=p.Ws, Tc=p.Tc, To=p.To, causal=p.causal)
    torch.cuda.synchronize()
    return y.cpu()


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("per_slab", [1, 2, 0])
def test_host_pipeline_equals_device_forward(dtype, causal, per_slab):
    # B = 2, h = 3: with 1 or 2 heads per slab there are 6 or 4 slabs (slots
    # reused), with 2 the last group of each batch element has one head.
    p = make_problem(batch=2, heads=3, T=5, Hs=7, Ws=9, D=128, Dp=128, Tc=2, To=1,
                     causal=causal, dtype=dtype, dist="scaled", seed=90 + per_slab)
    dev = device_tensors(p)
    ref = _device_y(p, dev)
    pin = per_slab != 1  # pageable host memory with one head per slab
    host = {n: (dev[n].cpu().pin_memory() if pin else dev[n].cpu()) for n in ("q", "k", "v")}
    y = rh.hybrid_attn_host(host["q"], host["k"], host["v"], dev["Wq"], dev["bq"], dev["Wk"],
                            dev["bk"], T=p.T, Hs=p.Hs, Ws=p.Ws, Tc=p.Tc, To=p.To,
                            causal=p.causal, heads_per_slab=per_slab)
    assert torch.equal(y, ref)


@pytest.mark.parametrize("per_slab", [3, 4])
def test_host_pipeline_uneven_slabs(per_slab):
    # B = 2, h = 5: the call's first and last slabs take ceil(per_slab / 2)
    # heads, the others per_slab or the rest of a batch element's heads.
    p = make_problem(batch=2, heads=5, T=4, Hs=6, Ws=11, D=128, Dp=128, Tc=2, To=1,
                     causal=False, dtype="bf16", dist="scaled", seed=95 + per_slab)
    dev = device_tensors(p)
    ref = _device_y(p, dev)
    host = {n: dev[n].cpu().pin_memory() for n in ("q", "k", "v")}
    y = rh.hybrid_attn_host(host["q"], host["k"], host["v"], dev["Wq"], dev["bq"], dev["Wk"],
                            dev["bk"], T=p.T, Hs=p.Hs, Ws=p.Ws, Tc=p.Tc, To=p.To,
                            causal=p.causal, heads_per_slab=per_slab)
    assert torch.equal(y, ref)


def test_host_pipeline_full_size_matches_device():
    """The bench layer (B = 2, h = 12, 21 x 30 x 52, bidirectional), two heads
    per slab, in the configuration the end-to-end measurement uses."""
    g = torch.Generator().manual_seed(5)
    B, H, T, Hs, Ws, D = 2, 12, 21, 30, 52, 128
    N = T * Hs * Ws
    q, k, v = ((torch.randn(B, H, N, D, generator=g) * 1.5).to(torch.bfloat16).pin_memory()
               for _ in range(3))
    Wq, Wk = ((0.1 * torch.randn(H, 2, D, 64, generator=g)).cuda() for _ in range(2))
    bq, bk = ((0.1 * torch.randn(H, 2, 64, generator=g)).cuda() for _ in range(2))
    kw = dict(T=T, Hs=Hs, Ws=Ws, Tc=3, To=1, causal=False)
    ref = rh.hybrid_attn(q.cuda(), k.cuda(), v.cuda(), Wq, bq, Wk, bk, **kw).cpu()
    y = rh.hybrid_attn_host(q, k, v, Wq, bq, Wk, bk, heads_per_slab=2, **kw)
    assert torch.equal(y, ref)


def test_host_pipeline_refuses_short_workspace():
    p = make_problem(batch=1, heads=2, T=3, Hs=4, Ws=4, D=128, Dp=128, Tc=1, To=0,
                     causal=False, dtype="bf16", seed=3)
    dev = device_tensors(p)
    params = rh.make_params(batch=1, heads=2, T=3, Hs=4, Ws=4, D=128, Dp=128, Tc=1, To=0,
                            causal=0, in_dtype=rh.BF16, out_dtype=rh.F32)
    need = rh.rehyat_host_workspace_bytes(params, 1)
    assert need > 0
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    h = {n: dev[n].cpu().pin_memory() for n in ("q", "k", "v")}
    y = torch.empty(1, 2, 48, 128, dtype=torch.float32).pin_memory()
    phi = rh.RehyatPhi(dev["Wq"].data_ptr(), dev["bq"].data_ptr(), dev["Wk"].data_ptr(),
                       dev["bk"].data_ptr())
    st = rh.rehyat_hybrid_attn_fwd_host(params, h["q"].data_ptr(), h["k"].data_ptr(),
                                        h["v"].data_ptr(), phi, y.data_ptr(), 1, ws.data_ptr(),
                                        need - 256, None)
    assert st == 4  # REHYAT_ERR_WORKSPACE


def test_host_pipeline_fp8_equals_device_fp8():
    """REHYAT_FLAG_FP8_QK through the host-buffer forward: each slab's forward
    makes its own E4M3 copies, bit-identical to the device fp8 forward."""
    p = make_problem(batch=2, heads=3, T=5, Hs=7, Ws=9, D=128, Dp=128, Tc=2, To=1,
                     causal=False, dtype="bf16", dist="scaled", seed=97)
    dev = device_tensors(p)
    kw = dict(T=p.T, Hs=p.Hs, Ws=p.Ws, Tc=p.Tc, To=p.To, causal=p.causal)
    ref = rh.hybrid_attn(dev["q"], dev["k"], dev["v"], dev["Wq"], dev["bq"], dev["Wk"],
                         dev["bk"], fp8_qk=True, **kw)
    torch.cuda.synchronize()
    host = {n: dev[n].cpu().pin_memory() for n in ("q", "k", "v")}
    y = rh.hybrid_attn_host(host["q"], host["k"], host["v"], dev["Wq"], dev["bq"], dev["Wk"],
                            dev["bk"], heads_per_slab=2, fp8_qk=True, **kw)
    assert torch.equal(y, ref.cpu())
