"""Helpers for the GPU parity tests: move a seeded problem to the device, run
it through the C ABI, and compare with the oracle at the stated tolerances.

Tolerances (y = the joint-normalised output):
  * fp32 inputs: max |y - y_oracle| <= 1e-5;
  * bf16 inputs (fp32 accumulation): max <= 2e-2 and mean <= 2e-3.
Branch partials are compared as normalised branch outputs (a^S/n^S and
a^L/n^L at the y tolerance), relative denominators, and the stabiliser c.
"""
import numpy as np
import torch

import linear_attention_video_chunked_b200 as rh

TOL = {"f32": dict(max=1e-5, mean=1e-5, rel=1e-5, c=1e-5),
       "bf16": dict(max=2e-2, mean=2e-3, rel=1e-2, c=1e-3)}


def device_tensors(p, device="cuda"):
    dt = torch.bfloat16 if p.dtype == "bf16" else torch.float32
    t = lambda a, d: torch.from_numpy(np.ascontiguousarray(a)).to(device=device, dtype=d)
    return dict(q=t(p.q, dt), k=t(p.k, dt), v=t(p.v, dt), Wq=t(p.Wq, torch.float32),
                bq=t(p.bq, torch.float32), Wk=t(p.Wk, torch.float32), bk=t(p.bk, torch.float32))


def run_fwd(p, *, debug=False, force_simt=False, one_tile=False, dev=None, out_dtype=None):
    dev = device_tensors(p) if dev is None else dev
    res = rh.hybrid_attn(dev["q"], dev["k"], dev["v"], dev["Wq"], dev["bq"], dev["Wk"], dev["bk"],
                         T=p.T, Hs=p.Hs, Ws=p.Ws, Tc=p.Tc, To=p.To, causal=p.causal,
                         debug=debug, force_simt=force_simt, one_tile=one_tile,
                         out_dtype=out_dtype)
    torch.cuda.synchronize()
    if debug:
        y, parts = res
        return (y.double().cpu().numpy(),
                {k: v.double().cpu().numpy() for k, v in parts.items()})
    return res.double().cpu().numpy()


def err_stats(y, ref):
    d = np.abs(np.asarray(y, np.float64) - np.asarray(ref, np.float64))
    return float(d.max()), float(d.mean())


def assert_close_y(y, ref, dtype, what="y"):
    tol = TOL[dtype]
    assert np.all(np.isfinite(y)), f"{what}: non-finite values"
    mx, mean = err_stats(y, ref)
    assert mx <= tol["max"], f"{what}: max abs err {mx:.3e} > {tol['max']}"
    assert mean <= tol["mean"], f"{what}: mean abs err {mean:.3e} > {tol['mean']}"
    return mx, mean


def assert_close_partials(parts, ref, dtype, rows=None):
    """Compare branch partials; ``rows`` optionally selects query rows."""
    tol = TOL[dtype]
    sel = (lambda a: a) if rows is None else (lambda a: a[..., rows, :] if a.ndim == 4 else a[..., rows])
    g = {k: sel(v) for k, v in parts.items()}
    r = {k: sel(np.asarray(v)) for k, v in ref.items()}
    assert_close_y(g["aS"] / g["nS"][..., None], r["aS"] / r["nS"][..., None], dtype, "aS/nS")
    rel_nS = np.abs(g["nS"] - r["nS"]) / r["nS"]
    assert rel_nS.max() <= tol["rel"], f"nS rel err {rel_nS.max():.3e}"
    dc = np.abs(g["c"] - r["c"]) / (1.0 + np.abs(r["c"]))
    assert dc.max() <= tol["c"], f"c err {dc.max():.3e}"
    has_lin = r["nL"] > 0
    if has_lin.any():
        rel_nL = np.abs(g["nL"] - r["nL"])[has_lin] / r["nL"][has_lin]
        assert rel_nL.max() <= tol["rel"], f"nL rel err {rel_nL.max():.3e}"
        aL = g["aL"][has_lin] / g["nL"][has_lin][..., None]
        aLr = r["aL"][has_lin] / r["nL"][has_lin][..., None]
        assert_close_y(aL, aLr, dtype, "aL/nL")
    assert np.all(g["nL"][~has_lin] == 0)
