"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on
the same seeded inputs.

Bars (y): fp32 inputs max abs <= 1e-5; bf16 inputs max abs <= 2e-2 and mean
abs <= 2e-3.  Branch partials are compared too, because at these feature-map
scales the linear branch carries most of the weight and would hide softmax
errors in y.
"""
import numpy as np
import pytest
import torch

import linear_attention_video_chunked_b200 as rh
from oracle import rehyat_oracle as orc
from rehyat_inputs import config_problem, make_problem
from tests.gpu_util import (assert_close_partials, assert_close_y, device_tensors, err_stats,
                            run_fwd)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    rh.lib()
    rh.rehyat_device_error_flags(reset=True)
    yield
    # No bounded wait inside the tensor-core kernels ran out during the module.
    assert rh.rehyat_device_error_flags() == 0


# ------------------------------------------------------------ tiny fp32 case
@pytest.mark.parametrize("causal", [False, True])
def test_tiny_fp32_both_forms(causal):
    p = config_problem("tiny_f32", causal=causal)
    ref_y, ref_p = orc.run_problem(p)
    y, parts = run_fwd(p, debug=True)
    assert_close_y(y, ref_y, "f32")
    assert_close_partials(parts, ref_p, "f32")


# ----------------------------------------- small ragged shapes, both dtypes
SMALL = [
    # B, h, T, Hs, Ws, D, Dp, Tc, To
    (1, 2, 5, 7, 9, 128, 128, 2, 1),     # HW=63: one ragged tile per slice
    (1, 2, 7, 10, 13, 128, 128, 3, 2),   # HW=130: tile straddles slices; T % Tc != 0
    (2, 1, 4, 16, 16, 128, 64, 1, 2),    # To > Tc, spatial-only chunks
    (1, 3, 6, 8, 12, 64, 256, 2, 0),     # no overlap, wide phi
    (1, 2, 3, 5, 5, 32, 32, 4, 1),       # one chunk covers everything
    (1, 1, 9, 11, 12, 128, 128, 3, 1),   # HW=132, several chunks
    (1, 2, 5, 9, 15, 128, 256, 2, 1),    # D'=256 on the tensor-core state path
    (1, 1, 40, 3, 4, 128, 64, 3, 1),     # long sequence of short slices (T = 40)
    (1, 1, 40, 3, 4, 128, 64, 5, 2),     # T = 40 in 8 chunks: the streaming chunk scan
]


@pytest.mark.parametrize("shape", SMALL, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("path", ["default", "simt", "one_tile"])
def test_small_shapes(shape, causal, dtype, path):
    """default = two-query-tile tensor-core kernel (bf16, D=128, D'<=128),
    one_tile = the one-tile tensor-core kernel, simt = fp32 CUDA cores."""
    B, h, T, Hs, Ws, D, Dp, Tc, To = shape
    if path == "one_tile" and dtype == "f32":
        pytest.skip("tensor-core kernels take bf16 inputs")
    p = make_problem(batch=B, heads=h, T=T, Hs=Hs, Ws=Ws, D=D, Dp=Dp, Tc=Tc, To=To,
                     causal=causal, dtype=dtype, dist="scaled", seed=100 + sum(shape))
    ref_y, ref_p = orc.run_problem(p)
    y, parts = run_fwd(p, debug=True, force_simt=path == "simt", one_tile=path == "one_tile")
    assert_close_y(y, ref_y, dtype)
    assert_close_partials(parts, ref_p, dtype)


def test_sharp_softmax_lowrank_inputs():
    """Low-rank-plus-noise q, k (logit std ~4) with a weak feature map, so the
    softmax branch dominates y."""
    p = make_problem(batch=1, heads=2, T=6, Hs=12, Ws=20, D=128, Dp=128, Tc=2, To=1,
                     causal=False, dtype="bf16", dist="lowrank", seed=77, phi_std=0.005)
    ref_y, ref_p = orc.run_problem(p)
    y, parts = run_fwd(p, debug=True)
    assert_close_y(y, ref_y, "bf16")
    assert_close_partials(parts, ref_p, "bf16")
    assert np.median(ref_p["nS"] / np.maximum(ref_p["nL"], 1e-30)) > 1.0


# ------------------------------------------------------- full-size workloads
def test_wan_320x480_causal_full():
    """Latent 21x20x30, 12 heads, D=128, T_c=3, T_o=1, causal, every output."""
    p = config_problem("wan_320x480_causal")
    ref_y, ref_p = orc.run_problem(p)
    y, parts = run_fwd(p, debug=True)
    assert_close_y(y, ref_y, "bf16")
    assert_close_partials(parts, ref_p, "bf16")


def test_wan_480x832_bidir_sampled_heads():
    """Latent 21x30x52, batch 2, 12 heads, bidirectional: every output of
    three sampled (batch, head) pairs against the oracle."""
    p = config_problem("wan_480x832_bidir")
    subset = [0, 13, 23]
    ref_y, ref_p = orc.run_problem(p, heads_subset=subset)
    y, parts = run_fwd(p, debug=True)
    B, H = p.batch, p.heads
    for idx in subset:
        b, hh = divmod(idx, H)
        assert_close_y(y[b, hh], ref_y[b, hh], "bf16", f"y[{b},{hh}]")
        assert_close_partials({k: v[b, hh] for k, v in parts.items()},
                              {k: v[b, hh] for k, v in ref_p.items()}, "bf16")
    assert np.all(np.isfinite(y))


@pytest.mark.parametrize("name,std,subset", [("wan_320x480_causal", 0.003, None),
                                             ("wan_480x832_bidir", 0.0045, [1, 5, 18])])
def test_balanced_branches_full_size(name, std, subset):
    """Feature-map scale chosen so the median n^L/n^S is near 1 on some heads
    (and far below on others): both branches are visible in y."""
    p = config_problem(name, phi_std=std)
    ref_y, ref_p = orc.run_problem(p, heads_subset=subset)
    y, parts = run_fwd(p, debug=True)
    for idx in (subset if subset is not None else range(p.batch * p.heads)):
        b, hh = divmod(idx, p.heads)
        assert_close_y(y[b, hh], ref_y[b, hh], "bf16", f"y[{b},{hh}]")
        assert_close_partials({k: v[b, hh] for k, v in parts.items()},
                              {k: v[b, hh] for k, v in ref_p.items()}, "bf16")


@pytest.mark.parametrize("causal", [False, True])
def test_wide_phi_several_items_per_cta(causal):
    """D'=256 with more (b*h, half, slice) items than SMs, so persistent
    state CTAs cross half and head boundaries and reload W_k mid-run."""
    p = make_problem(batch=1, heads=4, T=20, Hs=8, Ws=17, D=128, Dp=256, Tc=3, To=1,
                     causal=causal, dtype="bf16", dist="scaled", seed=77)
    ref_y, ref_p = orc.run_problem(p)
    y, parts = run_fwd(p, debug=True)
    assert_close_y(y, ref_y, "bf16")
    assert_close_partials(parts, ref_p, "bf16")


@pytest.mark.parametrize("Tc,To,Dp,causal", [(1, 0, 128, False), (2, 2, 64, True),
                                             (5, 1, 256, False), (7, 2, 128, True)])
def test_sweep_points_sampled(Tc, To, Dp, causal):
    """Points of the T_c / T_o / D' sweep on the 21x30x52 latent with
    low-rank-plus-noise q, k; one sampled head each."""
    p = make_problem(batch=1, heads=12, T=21, Hs=30, Ws=52, D=128, Dp=Dp, Tc=Tc, To=To,
                     causal=causal, dtype="bf16", dist="lowrank", seed=4 + Tc * 10 + To)
    subset = [5]
    ref_y, _ = orc.run_problem(p, heads_subset=subset)
    y = run_fwd(p)
    assert_close_y(y[0, 5], ref_y[0, 5], "bf16")


# ------------------------------------------------------------- comparator
def test_full_softmax_comparator():
    p = make_problem(batch=1, heads=2, T=3, Hs=10, Ws=30, D=128, Dp=32, Tc=1, To=0,
                     causal=False, dtype="bf16", seed=9)
    dev = device_tensors(p)
    y = rh.softmax_attn(dev["q"], dev["k"], dev["v"])
    torch.cuda.synchronize()
    ref = orc.full_softmax(p.q, p.k, p.v)
    assert_close_y(y.double().cpu().numpy(), ref, "bf16")


# ------------------------------------------------------------- streaming
def _stream_outputs(p, force_simt=False, dev=None):
    dev = device_tensors(p) if dev is None else dev
    st = rh.StreamingState(batch=p.batch, heads=p.heads, Hs=p.Hs, Ws=p.Ws, D=p.D, Dp=p.Dp,
                           Tc=p.Tc, To=p.To, Wq=dev["Wq"], bq=dev["bq"], Wk=dev["Wk"],
                           bk=dev["bk"], in_dtype=dev["q"].dtype, force_simt=force_simt)
    outs = []
    HW = p.HW
    for first in range(0, p.T, p.Tc):
        rows = slice(first * HW, min(p.T, first + p.Tc) * HW)
        qc, kc, vc = (dev[x][:, :, rows].contiguous() for x in ("q", "k", "v"))
        outs.append(st.step(qc, kc, vc))
    torch.cuda.synchronize()
    return torch.cat(outs, dim=2), st


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("Tc,To", [(3, 1), (2, 3), (1, 0), (4, 2)])
def test_streaming_matches_rnn_oracle_and_full_causal(dtype, Tc, To):
    p = make_problem(batch=1, heads=2, T=10, Hs=6, Ws=11, D=128, Dp=128, Tc=Tc, To=To,
                     causal=True, dtype=dtype, seed=31 + Tc + 7 * To)
    y_stream, _ = _stream_outputs(p)
    ref_y, _ = orc.run_problem(p, form="rnn")
    assert_close_y(y_stream.double().cpu().numpy(), ref_y, dtype)
    y_full = run_fwd(p)
    mx, _ = err_stats(y_stream.double().cpu().numpy(), y_full)
    assert mx <= (2e-2 if dtype == "bf16" else 1e-5)


@pytest.mark.parametrize("Dp,Tc,To", [(256, 3, 1), (64, 2, 2)])
def test_streaming_wide_and_narrow_phi(Dp, Tc, To):
    """The streaming fold on the tensor-core state kernel with D' = 256
    (two 128-feature halves per leaving slice) and D' = 64."""
    p = make_problem(batch=1, heads=3, T=11, Hs=9, Ws=15, D=128, Dp=Dp, Tc=Tc, To=To,
                     causal=True, dtype="bf16", seed=57 + Dp + Tc)
    y_stream, _ = _stream_outputs(p)
    ref_y, _ = orc.run_problem(p, form="rnn")
    assert_close_y(y_stream.double().cpu().numpy(), ref_y, "bf16")


@pytest.mark.parametrize("Tc,To,T", [(3, 1, 10), (2, 2, 7), (4, 0, 9)])
def test_streaming_split_key_window(Tc, To, T):
    """Chunks of 16x20 slices on 2 heads: the step splits each pair of query
    tiles' key window over several CTAs (the last chunk is one slice, split
    or not by its own schedule, and at T_c = 2 every chunk ends in a pair with
    tile A only, which runs whole).
    Outputs against the RNN oracle and the full causal forward, and bit for
    bit the same on a second run (the merge sums the pieces in order)."""
    p = make_problem(batch=1, heads=2, T=T, Hs=16, Ws=20, D=128, Dp=128, Tc=Tc, To=To,
                     causal=True, dtype="bf16", seed=71 + Tc + 5 * To)
    dev = device_tensors(p)
    y_stream, st = _stream_outputs(p, dev=dev)
    assert rh.rehyat_step_key_split(st.p, Tc) > 1
    ref_y, _ = orc.run_problem(p, form="rnn")
    assert_close_y(y_stream.double().cpu().numpy(), ref_y, "bf16")
    y_full = run_fwd(p)
    mx, _ = err_stats(y_stream.double().cpu().numpy(), y_full)
    assert mx <= 2e-2
    y_again, _ = _stream_outputs(p, dev=dev)
    assert torch.equal(y_again, y_stream)


def test_stream_81_slices_constant_memory():
    """81 slices of 30x52, 27 steps: outputs of sampled heads match the oracle
    and free device memory does not move across steps."""
    p = config_problem("stream_81x30x52")
    dev = device_tensors(p)
    st = rh.StreamingState(batch=p.batch, heads=p.heads, Hs=p.Hs, Ws=p.Ws, D=p.D, Dp=p.Dp,
                           Tc=p.Tc, To=p.To, Wq=dev["Wq"], bq=dev["bq"], Wk=dev["Wk"],
                           bk=dev["bk"], in_dtype=dev["q"].dtype)
    HW, rows_per = p.HW, p.Tc * p.HW
    chunks = [tuple(dev[x][:, :, s * rows_per:(s + 1) * rows_per].contiguous()
                    for x in ("q", "k", "v")) for s in range(27)]
    out = torch.empty(1, p.heads, rows_per, p.D, device="cuda")
    ys = []
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    frees = []
    # Head 3's pairs of query tiles run whole, head 10's as split key pieces
    # (the step's work list puts the pairs past the first wave in pieces).
    subset = [3, 10]
    for s in range(27):
        st.step(*chunks[s], out=out)
        ys.append(out[0, subset].double().cpu().numpy())
        frees.append(torch.cuda.mem_get_info()[0])
    assert all(f == free0 for f in frees)
    ref_y, _ = orc.run_problem(p, heads_subset=subset)
    got = np.concatenate(ys, axis=1)
    for i, h in enumerate(subset):
        assert_close_y(got[i], ref_y[0, h], "bf16")


# 16x20 slices: the step splits the key window (the arrival counters live in
# the state and return to zero every step).
@pytest.mark.parametrize("Hs,Ws", [(6, 11), (16, 20)])
def test_streaming_cuda_graph_replay_matches_eager(Hs, Ws):
    """One captured step replayed per chunk equals the eager steps bit for
    bit (the slice counter is read on the device)."""
    p = make_problem(batch=1, heads=2, T=10, Hs=Hs, Ws=Ws, D=128, Dp=128, Tc=2, To=1,
                     causal=True, dtype="bf16", seed=43)
    y_eager, st = _stream_outputs(p)
    dev = device_tensors(p)
    st.reset()
    HW, rows = p.HW, p.Tc * p.HW
    qb, kb, vb = (torch.empty(1, 2, rows, 128, device="cuda", dtype=torch.bfloat16)
                  for _ in range(3))
    out = torch.empty(1, 2, rows, 128, device="cuda")
    graph = st.capture_step(qb, kb, vb, out)
    outs = []
    for i in range(p.T // p.Tc):
        sl = slice(i * rows, (i + 1) * rows)
        qb.copy_(dev["q"][:, :, sl])
        kb.copy_(dev["k"][:, :, sl])
        vb.copy_(dev["v"][:, :, sl])
        graph.replay()
        outs.append(out.clone())
    torch.cuda.synchronize()
    assert torch.equal(torch.cat(outs, dim=2), y_eager)


@pytest.mark.parametrize("Hs,Ws", [(6, 11), (16, 20)])
def test_streaming_sequence_graph_matches_eager(Hs, Ws):
    """All steps of a stream captured as one CUDA graph (each step on its own
    chunk tensors) and replayed once give the eager outputs bit for bit, and
    a second replay after a reset gives them again."""
    p = make_problem(batch=1, heads=2, T=10, Hs=Hs, Ws=Ws, D=128, Dp=128, Tc=2, To=1,
                     causal=True, dtype="bf16", seed=43)
    y_eager, st = _stream_outputs(p)
    dev = device_tensors(p)
    rows = p.Tc * p.HW
    chunks = [tuple(dev[n][:, :, i * rows:(i + 1) * rows].contiguous() for n in "qkv")
              for i in range(p.T // p.Tc)]
    st.reset()
    out = torch.empty(1, 2, rows, 128, device="cuda")
    graph = st.capture_steps(chunks, out)
    for _ in range(2):
        st.reset()
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, y_eager[:, :, -rows:])


@pytest.mark.parametrize("Hs,Ws", [(6, 11), (16, 20)])
def test_streaming_checkpoint_resume_bit_exact(Hs, Ws):
    p = make_problem(batch=1, heads=2, T=9, Hs=Hs, Ws=Ws, D=128, Dp=128, Tc=2, To=1,
                     causal=True, dtype="bf16", seed=41)
    dev = device_tensors(p)
    mk = lambda: rh.StreamingState(batch=1, heads=2, Hs=Hs, Ws=Ws, D=128, Dp=128, Tc=2, To=1,
                                   Wq=dev["Wq"], bq=dev["bq"], Wk=dev["Wk"], bk=dev["bk"],
                                   in_dtype=torch.bfloat16)
    HW = p.HW
    chunk = lambda i: tuple(dev[x][:, :, i * 2 * HW:min(9, i * 2 + 2) * HW].contiguous()
                            for x in ("q", "k", "v"))
    a = mk()
    ya = [a.step(*chunk(i)).clone() for i in range(5)]
    b = mk()
    for i in range(2):
        b.step(*chunk(i))
    saved = b.snapshot().cpu()
    b.reset()
    b.step(*chunk(0))  # disturb
    b.restore(saved.cuda())
    yb = [b.step(*chunk(i)).clone() for i in range(2, 5)]
    torch.cuda.synchronize()
    for i in range(3):
        assert torch.equal(ya[2 + i], yb[i])


# ------------------------------------------------------------- properties
def test_repeatable_bitwise():
    p = config_problem("wan_320x480_causal")
    dev = device_tensors(p)
    y1 = run_fwd(p, dev=dev)
    y2 = run_fwd(p, dev=dev)
    assert np.array_equal(y1, y2)


def test_nan_input_propagates_without_fault():
    p = make_problem(batch=1, heads=1, T=4, Hs=4, Ws=8, D=64, Dp=64, Tc=2, To=1,
                     causal=True, dtype="bf16", seed=3)
    dev = device_tensors(p)
    dev["v"][0, 0, 5, 0] = float("nan")
    y = run_fwd(p, dev=dev)
    # slice 0 (rows 0..31) reaches every query, through the softmax window
    # (chunk 0) or the linear state (chunk 1); only value column 0 is NaN.
    assert np.isnan(y[0, 0, :, 0]).all()
    assert np.isfinite(y[0, 0, :, 1:]).all()


def test_bf16_output():
    p = make_problem(batch=1, heads=2, T=5, Hs=7, Ws=9, D=128, Dp=128, Tc=2, To=1,
                     causal=False, dtype="bf16", seed=8)
    ref_y, _ = orc.run_problem(p)
    y = run_fwd(p, out_dtype=torch.bfloat16)
    mx, mean = err_stats(y, ref_y)
    # bf16 output adds up to half an ulp of |y| on top of the fp32 result
    assert mean <= 2e-3 and mx <= 2e-2 + np.abs(ref_y).max() * 2.0 ** -8
