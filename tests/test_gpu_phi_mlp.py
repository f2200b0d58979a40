"""GPU parity of the general feature map (rehyat_feature_map_mlp) and of the
forward with given feature maps (rehyat_hybrid_attn_fwd_phi), through the C
ABI, against the fp64 oracle (oracle/rehyat_phi_mlp.py) on the same seeded
inputs.  Bars as for the forward: fp32 inputs max abs <= 1e-5 on y; bf16
inputs max abs <= 2e-2, mean abs <= 2e-3.  The feature map itself: on CUDA
cores (fp32) within 1e-5 relative to its largest value; on the tensor cores
(bf16 operands) within the first-order bound of rounding W_a, GELU(.) and
W_b to bf16 (unit roundoff u = 2^-8), element by element:
  |d psi_f| <= u * sum_j |W_b[j,f]| (1.13 sum_d |x_d W_a[d,j]| + 2 |g_j|),
  |d phi|   <= (|psi| + |d psi|)^i - |psi|^i   for part i,
with 1.13 >= max |GELU'|, times 1.1 for second-order and fp32 terms.
"""
import numpy as np
import pytest
import torch

import linear_attention_video_chunked_b200 as rh
from oracle import rehyat_oracle as orc
from oracle.rehyat_phi_mlp import feature_map_mlp, hybrid_phi_given
from rehyat_inputs import make_problem
from tests.gpu_util import assert_close_partials, assert_close_y, device_tensors
from tests.mlp_bound import bf16_bound

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    rh.lib()
    rh.rehyat_device_error_flags(reset=True)
    yield
    assert rh.rehyat_device_error_flags() == 0


def _mlp_params(H, D, Dh, Dp, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    Wa = rng.standard_normal((H, D, Dh)) / np.sqrt(D)
    ba = rng.standard_normal((H, Dh)) * 0.1
    Wb = rng.standard_normal((H, Dh, Dp)) / np.sqrt(Dh) * scale
    bb = rng.standard_normal((H, Dp)) * 0.1 * scale
    return [a.astype(np.float32) for a in (Wa, ba, Wb, bb)]


def _oracle_phi(x, params, parts):
    B, H = x.shape[:2]
    Wa, ba, Wb, bb = params
    return np.stack([np.stack([feature_map_mlp(x[b, h], Wa[h], ba[h], Wb[h], bb[h], parts)
                               for h in range(H)]) for b in range(B)])


def _cuda32(a):
    return torch.tensor(np.asarray(a, np.float32), device="cuda").contiguous()


@pytest.mark.parametrize("parts,dtype", [(1, "f32"), (2, "f32"), (4, "bf16")])
def test_feature_map_mlp_matches_oracle(parts, dtype):
    p = make_problem(batch=2, heads=3, T=3, Hs=5, Ws=7, D=64, Dp=128, Tc=1, To=0, causal=False,
                     dtype=dtype, seed=70 + parts)
    params = _mlp_params(3, 64, 96, 128, 71 + parts)
    dev = device_tensors(p)
    got = rh.feature_map_mlp(dev["q"], *(_cuda32(a) for a in params), parts=parts, T=p.T,
                             Hs=p.Hs, Ws=p.Ws)
    torch.cuda.synchronize()
    ref = _oracle_phi(np.asarray(p.q, np.float64), params, parts)
    err = np.abs(got.double().cpu().numpy() - ref).max()
    assert err <= 1e-5 * np.abs(ref).max(), err


def _closed_form_phi(p):
    fq = np.stack([np.stack([orc.feature_map(p.q[b, h], p.Wq[h], p.bq[h])
                             for h in range(p.heads)]) for b in range(p.batch)])
    fk = np.stack([np.stack([orc.feature_map(p.k[b, h], p.Wk[h], p.bk[h])
                             for h in range(p.heads)]) for b in range(p.batch)])
    return fq.astype(np.float32), fk.astype(np.float32)


def _run_phi(p, fq, fk, force_simt):
    dev = device_tensors(p)
    y, parts = rh.hybrid_attn_phi(dev["q"], dev["k"], dev["v"], _cuda32(fq), _cuda32(fk), T=p.T,
                                  Hs=p.Hs, Ws=p.Ws, Tc=p.Tc, To=p.To, causal=p.causal,
                                  debug=True, force_simt=force_simt)
    torch.cuda.synchronize()
    return y.double().cpu().numpy(), {k: v.double().cpu().numpy() for k, v in parts.items()}


SHAPES = [
    # B, h, T, Hs, Ws, D, Dp, Tc, To, causal
    (1, 2, 5, 7, 9, 128, 128, 2, 1, False),    # ragged tiles
    (1, 2, 7, 10, 13, 128, 64, 3, 2, True),
    (1, 2, 5, 9, 15, 128, 256, 2, 1, False),   # D' = 256: state halves, two readout pieces
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_phi_given_closed_form(shape, dtype):
    """Closed-form phi passed as arrays: equals the oracle's phi-given forward
    (itself pinned to the closed-form forward)."""
    B, h, T, Hs, Ws, D, Dp, Tc, To, causal = shape
    p = make_problem(batch=B, heads=h, T=T, Hs=Hs, Ws=Ws, D=D, Dp=Dp, Tc=Tc, To=To,
                     causal=causal, dtype=dtype, dist="scaled", seed=400 + sum(shape[:9]))
    fq, fk = _closed_form_phi(p)
    ref_y, ref_p = hybrid_phi_given(p.q, p.k, p.v, fq, fk, T=p.T, HW=p.HW, Tc=p.Tc, To=p.To,
                                    causal=p.causal)
    y, parts = _run_phi(p, fq, fk, force_simt=dtype == "f32")
    assert_close_y(y, ref_y, dtype)
    assert_close_partials(parts, ref_p, dtype)


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_phi_given_bf16_maps(shape, dtype):
    """The maps given in bf16 (REHYAT_FLAG_PHI_BF16): equals the oracle's
    phi-given forward on the same bf16-rounded maps."""
    B, h, T, Hs, Ws, D, Dp, Tc, To, causal = shape
    p = make_problem(batch=B, heads=h, T=T, Hs=Hs, Ws=Ws, D=D, Dp=Dp, Tc=Tc, To=To,
                     causal=causal, dtype=dtype, dist="scaled", seed=450 + sum(shape[:9]))
    fq, fk = _closed_form_phi(p)
    fq16, fk16 = (_cuda32(f).to(torch.bfloat16) for f in (fq, fk))
    rq, rk = (f.double().cpu().numpy() for f in (fq16, fk16))
    ref_y, ref_p = hybrid_phi_given(p.q, p.k, p.v, rq, rk, T=p.T, HW=p.HW, Tc=p.Tc, To=p.To,
                                    causal=p.causal)
    dev = device_tensors(p)
    y, parts = rh.hybrid_attn_phi(dev["q"], dev["k"], dev["v"], fq16, fk16, T=p.T, Hs=p.Hs,
                                  Ws=p.Ws, Tc=p.Tc, To=p.To, causal=p.causal, debug=True,
                                  force_simt=dtype == "f32")
    torch.cuda.synchronize()
    assert_close_y(y.double().cpu().numpy(), ref_y, dtype)
    assert_close_partials({k: v.double().cpu().numpy() for k, v in parts.items()}, ref_p, dtype)


@pytest.mark.parametrize("force_simt", [False, True])
def test_feature_map_mlp_bf16_output_is_the_rounded_fp32_map(force_simt):
    """REHYAT_FLAG_PHI_BF16 rounds the map the fp32 output holds (same
    arithmetic, round to nearest even at the store): bit for bit."""
    p = make_problem(batch=2, heads=2, T=3, Hs=7, Ws=9, D=128, Dp=128, Tc=1, To=0,
                     causal=False, dtype="bf16", seed=77)
    params = [_cuda32(a) for a in _mlp_params(2, 128, 256, 128, 78, scale=0.5)]
    dev = device_tensors(p)
    kw = dict(parts=2, T=p.T, Hs=p.Hs, Ws=p.Ws, force_simt=force_simt)
    f32 = rh.feature_map_mlp(dev["q"], *params, **kw)
    b16 = rh.feature_map_mlp(dev["q"], *params, out_dtype=torch.bfloat16, **kw)
    torch.cuda.synchronize()
    assert b16.dtype == torch.bfloat16
    assert torch.equal(b16, f32.to(torch.bfloat16))


@pytest.mark.parametrize("dtype,parts_n", [("bf16", 2), ("f32", 2), ("bf16", 4)])
@pytest.mark.parametrize("causal", [False, True])
def test_mlp_phi_end_to_end(dtype, parts_n, causal):
    """General phi (a degree-1 part, so negative values) from the library's
    MLP kernel through the phi-given forward, against the oracle."""
    p = make_problem(batch=1, heads=2, T=6, Hs=8, Ws=12, D=128, Dp=128, Tc=2, To=1,
                     causal=causal, dtype=dtype, dist="scaled", seed=500 + parts_n)
    params = _mlp_params(2, 128, 384, 128, 501, scale=0.5)
    dev = device_tensors(p)
    kw = dict(T=p.T, Hs=p.Hs, Ws=p.Ws)
    pq = rh.feature_map_mlp(dev["q"], *(_cuda32(a) for a in params), parts=parts_n, **kw)
    pk = rh.feature_map_mlp(dev["k"], *(_cuda32(a) for a in params), parts=parts_n, **kw)
    y, parts = rh.hybrid_attn_phi(dev["q"], dev["k"], dev["v"], pq, pk, Tc=p.Tc, To=p.To,
                                  causal=p.causal, debug=True, force_simt=dtype == "f32", **kw)
    torch.cuda.synchronize()
    fq = _oracle_phi(np.asarray(p.q, np.float64), params, parts_n)
    fk = _oracle_phi(np.asarray(p.k, np.float64), params, parts_n)
    assert fq.min() < 0 and fk.min() < 0  # the degree-1 part is signed
    ref_y, ref_p = hybrid_phi_given(p.q, p.k, p.v, fq, fk, T=p.T, HW=p.HW, Tc=p.Tc, To=p.To,
                                    causal=p.causal)
    assert_close_y(y.double().cpu().numpy(), ref_y, dtype)
    # The linear partials are signed here: compare them against their scale.
    got = {k: v.double().cpu().numpy() for k, v in parts.items()}
    assert_close_y(got["aS"] / got["nS"][..., None], ref_p["aS"] / ref_p["nS"][..., None], dtype,
                   "aS/nS")
    rel = 1e-5 if dtype == "f32" else 2e-2
    for key in ("nL", "aL"):
        err = np.abs(got[key] - ref_p[key]).max()
        assert err <= rel * np.abs(ref_p[key]).max(), (key, err)


# ------------------------------------------------ tensor-core feature map
def _tc_map(x_dev, params, parts, T, Hs, Ws):
    """phi (fp32 CUDA tensor) from the tensor-core path of the C ABI."""
    B, H, N, D = x_dev.shape
    Dh, Dp = params[0].shape[-1], params[2].shape[-1]
    p = rh.make_params(batch=B, heads=H, T=T, Hs=Hs, Ws=Ws, D=D, Dp=Dp, Tc=1, To=0, causal=0,
                       in_dtype=rh.BF16, out_dtype=rh.F32)
    dev = [_cuda32(t) for t in params]
    phi = torch.empty(B, H, N, Dp, dtype=torch.float32, device="cuda")
    mlp = rh.RehyatPhiMlp(*(t.data_ptr() for t in dev), Dh, parts)
    nbytes = rh.rehyat_feature_map_mlp_workspace_bytes(p, mlp, x_dev.data_ptr(), phi.data_ptr())
    assert nbytes > 0, "tensor-core path not selected"
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    st = rh.rehyat_feature_map_mlp(p, x_dev.data_ptr(), mlp, phi.data_ptr(), ws.data_ptr(),
                                   nbytes, torch.cuda.current_stream().cuda_stream)
    assert st == 0, rh.rehyat_status_string(st)
    # Too small a workspace is refused before any launch.
    assert rh.rehyat_feature_map_mlp(p, x_dev.data_ptr(), mlp, phi.data_ptr(), ws.data_ptr(),
                                     nbytes - 16, None) == 4  # REHYAT_ERR_WORKSPACE
    torch.cuda.synchronize()
    return phi


TC_SHAPES = [
    # B, h, T, Hs, Ws, Dh, Dp, parts: what it covers
    (1, 2, 1, 5, 19, 128, 128, 2),     # N = 95 < 128: one ragged tile per (b,h)
    (1, 3, 1, 43, 179, 384, 128, 2),   # 61 tiles per head: a CTA of 2 tiles spans two heads
    (2, 4, 2, 9, 289, 256, 64, 4),     # 41 tiles per (b,h), 3 per CTA; D' = 64, P = 4
    (1, 2, 3, 7, 13, 512, 64, 1),      # D_h = 512 (largest that fits with D' = 64), P = 1
]


@pytest.mark.parametrize("shape", TC_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_feature_map_mlp_tensor_cores_withinbf16_bound(shape):
    B, H, T, Hs, Ws, Dh, Dp, parts = shape
    p = make_problem(batch=B, heads=H, T=T, Hs=Hs, Ws=Ws, D=128, Dp=Dp, Tc=1, To=0,
                     causal=False, dtype="bf16", seed=600 + Dh + parts)
    params = _mlp_params(H, 128, Dh, Dp, 601 + Dh, scale=0.5)
    got = _tc_map(device_tensors(p)["q"], params, parts, T, Hs, Ws).double().cpu().numpy()
    Wa, ba, Wb, bb = params
    x = np.asarray(p.q, np.float64)
    for b in range(B):
        for h in range(H):
            ref = feature_map_mlp(x[b, h], Wa[h], ba[h], Wb[h], bb[h], parts)
            bound = bf16_bound(x[b, h], Wa[h], ba[h], Wb[h], bb[h], parts)
            err = np.abs(got[b, h] - ref)
            worst = np.unravel_index(np.argmax(err - bound), err.shape)
            assert np.all(err <= bound + 1e-6 * np.abs(ref).max()), (b, h, worst, err[worst],
                                                                       bound[worst])
            # The bound is not vacuous: the typical error is far inside it.
            assert np.median(err) < 0.25 * np.median(bound) + 1e-12


def test_feature_map_mlp_tensor_cores_full_size_sampled_rows():
    """The general-phi bench configuration (B = 2, h = 12, 21 x 30 x 52,
    D_h = 3D = 384, D' = 128, P = 2) in the launch the bench times, checked
    on 64 sampled tokens of every (b, h) against the oracle."""
    B, H, T, Hs, Ws, Dh, Dp, parts = 2, 12, 21, 30, 52, 384, 128, 2
    N = T * Hs * Ws
    g = torch.Generator().manual_seed(7)
    x = (torch.randn(B, H, N, 128, generator=g) * 1.5).to(torch.bfloat16)
    params = _mlp_params(H, 128, Dh, Dp, 602, scale=0.5)
    rows = np.random.default_rng(8).choice(N, size=64, replace=False)
    rows[:2] = [0, N - 1]
    idx = torch.tensor(rows)
    got = _tc_map(x.cuda(), params, parts, T, Hs, Ws)[:, :, idx.cuda()].double().cpu().numpy()
    xs = x[:, :, idx].double().numpy()
    Wa, ba, Wb, bb = params
    for b in range(B):
        for h in range(H):
            xr = xs[b, h]
            ref = feature_map_mlp(xr, Wa[h], ba[h], Wb[h], bb[h], parts)
            bound = bf16_bound(xr, Wa[h], ba[h], Wb[h], bb[h], parts)
            err = np.abs(got[b, h] - ref)
            assert np.all(err <= bound + 1e-6 * np.abs(ref).max()), (b, h, err.max())


def test_feature_map_mlp_force_simt_and_fp32_take_cuda_cores():
    """FLAG_FORCE_SIMT (and fp32 x) select the fp32 CUDA-core kernel, which
    needs no workspace and meets the fp32 bar."""
    p = make_problem(batch=1, heads=2, T=2, Hs=5, Ws=7, D=128, Dp=128, Tc=1, To=0,
                     causal=False, dtype="bf16", seed=77)
    params = _mlp_params(2, 128, 256, 128, 78)
    dev = device_tensors(p)
    got = rh.feature_map_mlp(dev["q"], *(_cuda32(a) for a in params), parts=2, T=p.T, Hs=p.Hs,
                             Ws=p.Ws, force_simt=True)
    torch.cuda.synchronize()
    ref = _oracle_phi(np.asarray(p.q, np.float64), params, 2)
    err = np.abs(got.double().cpu().numpy() - ref).max()
    assert err <= 1e-5 * np.abs(ref).max(), err
    pf = rh.make_params(batch=1, heads=2, T=p.T, Hs=p.Hs, Ws=p.Ws, D=128, Dp=128, Tc=1, To=0,
                        causal=0, in_dtype=rh.F32, out_dtype=rh.F32)
    mlp = rh.RehyatPhiMlp(*(_cuda32(a).data_ptr() for a in params), 256, 2)
    assert rh.rehyat_feature_map_mlp_workspace_bytes(pf, mlp, dev["q"].data_ptr(),
                                                     got.data_ptr()) == 0


def test_feature_map_mlp_tensor_cores_gelu_identity_weights():
    """W_a = W_b = I (exact in bf16), one part: psi = bf16(GELU(x + b_a)) + b_b,
    so the kernel's GELU is seen directly: within one bf16 rounding (2^-8
    relative) of the exact GELU plus 1e-6 |u| for its erf approximation
    (Abramowitz & Stegun 7.1.28, 3e-7) and its fp32 evaluation."""
    B, H, T, Hs, Ws = 1, 2, 1, 16, 40
    N = T * Hs * Ws
    g = torch.Generator().manual_seed(11)
    x = (torch.randn(B, H, N, 128, generator=g) * 3.0).to(torch.bfloat16)
    eye = np.stack([np.eye(128)] * H)
    rng = np.random.default_rng(12)
    ba = rng.standard_normal((H, 128)) * 0.5
    bb = rng.standard_normal((H, 128)) * 0.1
    params = [a.astype(np.float32) for a in (eye, ba, eye, bb)]
    got = _tc_map(x.cuda(), params, 1, T, Hs, Ws).double().cpu().numpy()
    u = (x.double().numpy() + params[1].astype(np.float64)[None, :, None, :]).astype(np.float32)
    u = u.astype(np.float64)
    from scipy.special import erf
    gl = 0.5 * u * (1.0 + erf(u / np.sqrt(2.0)))
    err = np.abs(got - params[3].astype(np.float64)[None, :, None, :] - gl)
    bar = 2.0 ** -8 * np.abs(gl) + 1e-6 * np.maximum(1.0, np.abs(u))
    assert np.all(err <= bar), float((err - bar).max())
    assert (u < -3).any() and (u > 3).any()


@pytest.mark.parametrize("force_simt", [False, True])
def test_denominator_report_counts_cancelled_rows(force_simt):
    """A signed phi_q that drives n^S + n^L below zero on chosen rows: the
    forward keeps y as the formula gives it and the report counts exactly
    those rows (tensor-core and CUDA-core kernels)."""
    p = make_problem(batch=1, heads=2, T=4, Hs=8, Ws=8, D=128, Dp=64, Tc=1, To=0,
                     causal=False, dtype="bf16", seed=31)
    dev = device_tensors(p)
    B, H, N = 1, 2, p.N
    fk = torch.full((B, H, N, 64), 0.01, dtype=torch.float32, device="cuda")
    fq = torch.full((B, H, N, 64), 0.01, dtype=torch.float32, device="cuda")
    bad = torch.zeros(B, H, N, dtype=torch.bool, device="cuda")
    bad[0, 0, 5:17] = True
    bad[0, 1, 100:103] = True
    # n^L = phi_q . z_L with z_L = 0.01 * 64 * (keys in the linear set) > 0:
    # a large negative phi_q on the chosen rows makes n^S + n^L < 0.
    fq[bad] = -1e3
    rh.rehyat_denominator_report(reset=True)
    y, parts = rh.hybrid_attn_phi(dev["q"], dev["k"], dev["v"], fq, fk, T=p.T, Hs=p.Hs, Ws=p.Ws,
                                  Tc=p.Tc, To=p.To, causal=p.causal, debug=True,
                                  force_simt=force_simt)
    torch.cuda.synchronize()
    den = parts["nS"] + parts["nL"]
    assert bool((den[bad] < 0).all()) and bool((den[~bad] > 0).all())
    assert rh.rehyat_denominator_report(reset=True) == int(bad.sum())
    assert rh.rehyat_denominator_report() == 0
    # The closed-form phi (squares) never adds to the count.
    rh.hybrid_attn(dev["q"], dev["k"], dev["v"], dev["Wq"], dev["bq"], dev["Wk"], dev["bk"],
                   T=p.T, Hs=p.Hs, Ws=p.Ws, Tc=p.Tc, To=p.To, causal=p.causal,
                   force_simt=force_simt)
    torch.cuda.synchronize()
    assert rh.rehyat_denominator_report() == 0
