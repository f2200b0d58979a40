"""Host-side checks of the C ABI (no GPU needed).

The library loads, exports every function include/rehyat.h declares, sizes
its workspace/state correctly, and rejects bad arguments with a status before
launching anything.
"""
import ctypes
import os
import re

import pytest

import linear_attention_video_chunked_b200 as rh

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "rehyat.h")


def _declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"REHYAT_API\s+[\w\s\*]*?\b(rehyat_\w+)\s*\(", text)))


def _params(**kw):
    base = dict(batch=2, heads=3, T=7, Hs=5, Ws=6, D=128, Dp=128, Tc=3, To=1, causal=0,
                in_dtype=rh.BF16, out_dtype=rh.F32)
    base.update(kw)
    return rh.make_params(**base)


def test_library_loads_and_exports_every_declared_symbol():
    L = rh.lib()
    declared = _declared_functions()
    assert len(declared) >= 9
    for name in declared:
        assert hasattr(L, name), name
        assert ctypes.cast(getattr(L, name), ctypes.c_void_p).value
    assert set(declared) == set(rh.EXPORTED_SYMBOLS)
    assert rh.rehyat_version() >= 100


def test_attention_path_selection():
    assert rh.rehyat_attn_path(_params()) == 1                       # bf16, D=128, Dp=128
    assert rh.rehyat_attn_path(_params(Dp=64)) == 1
    assert rh.rehyat_attn_path(_params(Dp=256)) == 1
    assert rh.rehyat_attn_path(_params(Dp=32)) == 0                  # CUDA-core kernel
    assert rh.rehyat_attn_path(_params(D=64)) == 0
    assert rh.rehyat_attn_path(_params(in_dtype=rh.F32)) == 0
    assert rh.rehyat_attn_path(_params(flags=rh.FLAG_FORCE_SIMT)) == 0
    assert rh.rehyat_attn_path(_params(T=0)) == -1


def test_status_strings():
    for code in range(7):
        assert rh.rehyat_status_string(code) != "unknown status"
    assert rh.rehyat_status_string(0) == "ok"


def test_workspace_bytes_layout():
    p = _params()
    BH, T, Dp, D, nch = 6, 7, 128, 128, 3
    need = BH * T * Dp * D * 4 + BH * T * Dp * 4 + BH * nch * Dp * D * 4 + BH * nch * Dp * 4
    need += 2 * 3 * Dp * D * 2  # bf16 phi_q and phi_k weight images, per head
    got = rh.rehyat_workspace_bytes(p)
    assert need <= got <= need + 6 * 256
    assert got % 256 == 0


def test_state_bytes_constant_and_ring_sized_by_overlap():
    p1 = _params(causal=1, To=1)
    p2 = _params(causal=1, To=2)
    b1, b2 = rh.rehyat_state_bytes(p1), rh.rehyat_state_bytes(p2)
    ring_slice = 6 * 30 * 128 * 2 * 2  # BH * HW * D * bf16 * (k and v)
    assert abs((b2 - b1) - ring_slice) <= 512
    # independent of the number of slices in the video
    assert rh.rehyat_state_bytes(_params(causal=1, T=100)) == b1


@pytest.mark.parametrize("bad", [
    dict(batch=0), dict(heads=-1), dict(T=0), dict(Hs=0), dict(Tc=0), dict(To=-1),
    dict(causal=2), dict(in_dtype=7), dict(out_dtype=-1), dict(scale=-1.0),
    dict(scale=float("nan")),
])
def test_invalid_params_rejected(bad):
    p = _params(**bad)
    assert rh.rehyat_workspace_bytes(p) == 0
    st = rh.rehyat_hybrid_attn_fwd(p, 16, 16, 16, rh.RehyatPhi(16, 16, 16, 16), 16, 16, 1 << 40,
                                   None, None)
    assert st == 1


@pytest.mark.parametrize("bad", [dict(D=96), dict(D=256), dict(Dp=48), dict(Dp=512)])
def test_unsupported_shapes_rejected(bad):
    p = _params(**bad)
    assert rh.rehyat_workspace_bytes(p) == 0
    st = rh.rehyat_hybrid_attn_fwd(p, 16, 16, 16, rh.RehyatPhi(16, 16, 16, 16), 16, 16, 1 << 40,
                                   None, None)
    assert st == 2


def test_pointer_checks_before_launch():
    p = _params()
    phi = rh.RehyatPhi(4096, 4096, 4096, 4096)
    ws = rh.rehyat_workspace_bytes(p)
    f = rh.rehyat_hybrid_attn_fwd
    assert f(p, 0, 4096, 4096, phi, 4096, 4096, ws, None, None) == 1       # null q
    assert f(p, 4096, 4096, 4096, rh.RehyatPhi(0, 4096, 4096, 4096), 4096, 4096, ws, None,
             None) == 1                                                    # null phi
    assert f(p, 4104, 4096, 4096, phi, 4096, 4096, ws, None, None) == 3    # misaligned q
    assert f(p, 4096, 4096, 4096, phi, 4096, 4096, ws - 1, None, None) == 4  # short ws
    dbg = rh.RehyatDebug(4098, 0, 0, 0, 0)
    assert f(p, 4096, 4096, 4096, phi, 4096, 4096, ws, dbg, None) == 3    # misaligned dbg


def test_chunk_step_argument_checks():
    p = _params(causal=1)
    phi = rh.RehyatPhi(4096, 4096, 4096, 4096)
    ws = rh.rehyat_step_workspace_bytes(p)
    step = rh.rehyat_chunk_step
    assert step(_params(causal=0), 4096, 4096, 4096, 1, phi, 4096, 4096, 4096, ws, None,
                None) == 1                                                 # not causal
    assert step(p, 4096, 4096, 4096, 0, phi, 4096, 4096, 4096, ws, None, None) == 1
    assert step(p, 4096, 4096, 4096, 4, phi, 4096, 4096, 4096, ws, None, None) == 1  # > Tc
    assert step(p, 4096, 4096, 4096, 2, phi, 0, 4096, 4096, ws, None, None) == 1     # state
    assert step(p, 4096, 4096, 4096, 2, phi, 4100, 4096, 4096, ws, None, None) == 3
    assert step(p, 4096, 4096, 4096, 2, phi, 4096, 4096, 4096, ws - 256, None, None) == 4
    assert rh.rehyat_state_init(p, 0, None) == 1
    assert rh.rehyat_state_init(p, 4104, None) == 3


def test_softmax_entry_checks():
    p = _params()
    assert rh.rehyat_softmax_attn_fwd(p, 0, 16, 16, 16, None) == 1
    assert rh.rehyat_softmax_attn_fwd(p, 24, 16, 16, 16, None) == 3


def test_split_stage_argument_checks():
    p = _params()
    phi = rh.RehyatPhi(4096, 4096, 4096, 4096)
    ws = rh.rehyat_workspace_bytes(p)
    state, attn = rh.rehyat_fwd_state, rh.rehyat_fwd_attn
    assert state(p, 0, 4096, phi, 4096, ws, None) == 1                  # null k
    assert state(p, 4096, 4096, rh.RehyatPhi(4096, 4096, 0, 4096), 4096, ws, None) == 1
    assert state(p, 4096, 4104, phi, 4096, ws, None) == 3               # misaligned v
    assert state(p, 4096, 4096, phi, 4096, ws - 1, None) == 4
    assert attn(p, 4096, 4096, 4096, phi, 0, 4096, ws, None, None) == 1  # null y
    assert attn(p, 4096, 4096, 4096, phi, 4096, 4100, ws, None, None) == 3
    assert attn(p, 4096, 4096, 4096, phi, 4096, 4096, ws - 1, None, None) == 4
    assert attn(_params(batch=0), 4096, 4096, 4096, phi, 4096, 4096, ws, None, None) == 1


def _mlp(parts=2, Dh=256, ptrs=(4096, 4096, 4096, 4096)):
    return rh.RehyatPhiMlp(*ptrs, Dh, parts)


def test_feature_map_argument_checks():
    p = _params()
    f = rh.rehyat_feature_map_mlp
    assert f(p, 4096, _mlp(parts=0), 4096, None, 0, None) == 1
    assert f(p, 4096, _mlp(parts=3), 4096, None, 0, None) == 1          # D' = 128 not in 3 parts
    assert f(p, 4096, _mlp(Dh=0), 4096, None, 0, None) == 1
    assert f(p, 4096, _mlp(Dh=640), 4096, None, 0, None) == 2           # D_h > 512
    assert f(p, 0, _mlp(), 4096, None, 0, None) == 1                    # null x
    assert f(p, 4096, _mlp(), 0, None, 0, None) == 1                    # null phi
    assert f(p, 4096, _mlp(ptrs=(4096, 0, 4096, 4096)), 4096, None, 0, None) == 1  # null b_a
    assert f(p, 4098, _mlp(), 4096, None, 0, None) == 3                 # x not 4-byte aligned
    assert f(p, 4096, _mlp(ptrs=(4096, 4096, 4096, 4097)), 4096, None, 0, None) == 3
    assert f(_params(T=0), 4096, _mlp(), 4096, None, 0, None) == 1
    # The fp8 flag belongs to the softmax branch of the full forward only.
    fp8 = _params(flags=rh.FLAG_FP8_QK)
    assert f(fp8, 4096, _mlp(), 4096, None, 0, None) == 2
    assert rh.rehyat_feature_map_mlp_workspace_bytes(fp8, _mlp(), 4096, 4096) == 0
    assert rh.rehyat_feature_map_mlp_workspace_bytes(p, _mlp(parts=0), 4096, 4096) == 0


def test_phi_given_forward_argument_checks():
    p = _params()
    ws = rh.rehyat_workspace_bytes(p)
    f = rh.rehyat_hybrid_attn_fwd_phi
    assert f(p, 4096, 4096, 4096, 0, 4096, 4096, 4096, ws, None, None) == 1     # null phi_q
    assert f(p, 4096, 4096, 4096, 4096, 0, 4096, 4096, ws, None, None) == 1     # null phi_k
    assert f(p, 4096, 4096, 4096, 4100, 4096, 4096, 4096, ws, None, None) == 3  # phi_q
    assert f(p, 4096, 4096, 4096, 4096, 4096, 4096, 4096, ws - 1, None, None) == 4
    dbg = rh.RehyatDebug(4096, 4098, 0, 0, 0)
    assert f(p, 4096, 4096, 4096, 4096, 4096, 4096, 4096, ws, dbg, None) == 3
    assert f(_params(flags=rh.FLAG_FP8_QK), 4096, 4096, 4096, 4096, 4096, 4096, 4096, ws,
             None, None) == 2


def test_phi_backward_argument_checks():
    p = _params()
    phi = rh.RehyatPhi(4096, 4096, 4096, 4096)
    grad = rh.RehyatPhiGrad(4096, 4096, 4096, 4096)
    ws = rh.rehyat_phi_bwd_workspace_bytes(p)
    assert ws > rh.rehyat_workspace_bytes(p)      # the forward's state plus the partials
    f = rh.rehyat_phi_bwd
    args = [p, 4096, 4096, 4096, 4096, 4096, 4096, phi, grad, 4096, ws, None]

    def call(**change):
        a = list(args)
        for i, val in change.items():
            a[int(i[1:])] = val
        return f(*a)

    assert call(a6=0) == 1                                               # null den
    assert call(a8=rh.RehyatPhiGrad(4096, 0, 4096, 4096)) == 1           # null db_q
    assert call(a7=rh.RehyatPhi(0, 4096, 4096, 4096)) == 1               # null W_q
    assert call(a5=4100) == 3                                            # dy not 16-byte aligned
    assert call(a6=4098) == 3                                            # den not 4-byte aligned
    assert call(a8=rh.RehyatPhiGrad(4096, 4096, 4097, 4096)) == 3
    assert call(a10=ws - 1) == 4
    assert call(a0=_params(flags=rh.FLAG_FP8_QK)) == 2
    assert rh.rehyat_phi_bwd_workspace_bytes(_params(flags=rh.FLAG_FP8_QK)) == 0
    assert rh.rehyat_phi_bwd_workspace_bytes(_params(heads=0)) == 0


C_PROGRAM = r"""
#include <stdio.h>
#include "rehyat.h"
int main(void) {
  rehyat_params p = {2, 12, 21, 30, 52, 128, 128, 3, 1, 0, REHYAT_BF16, REHYAT_F32, 0.0f, 0};
  rehyat_params bad = p;
  rehyat_status st;
  size_t ws = rehyat_workspace_bytes(&p);
  int path = rehyat_attn_path(&p);
  bad.T = 0;
  st = rehyat_hybrid_attn_fwd(&bad, NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL, NULL);
  printf("%d %zu %d %d\n", rehyat_version(), ws, path, (int)st);
  return 0;
}
"""


def test_full_backward_argument_checks():
    p = _params()
    phi = rh.RehyatPhi(4096, 4096, 4096, 4096)
    grad = rh.RehyatPhiGrad(4096, 4096, 4096, 4096)
    ws = rh.rehyat_hybrid_attn_bwd_workspace_bytes(p)
    rows = 2 * 3 * 7 * 5 * 6
    # The feature-map backward's workspace holds, for the tensor-core passes'
    # shapes, r and bf16 dy / den per row; the full backward shares them and
    # adds Dc and j*.
    ws_phi = rh.rehyat_phi_bwd_workspace_bytes(p)
    ws_phi_simt = rh.rehyat_phi_bwd_workspace_bytes(_params(flags=rh.FLAG_FORCE_SIMT))
    assert ws_phi - ws_phi_simt >= 4 * rows + 2 * 128 * rows
    assert ws - ws_phi >= 2 * 4 * rows
    f = rh.rehyat_hybrid_attn_bwd
    # p, q, k, v, phi, y, dy, c, den, dq, dk, dv, grad, workspace, ws_bytes, stream
    args = [p, 4096, 4096, 4096, phi, 4096, 4096, 4096, 4096, 4096, 4096, 4096, grad, 4096, ws,
            None]

    def call(**change):
        a = list(args)
        for i, val in change.items():
            a[int(i[1:])] = val
        return f(*a)

    assert call(a7=0) == 1                                               # null c
    assert call(a8=0) == 1                                               # null den
    assert call(a10=0) == 1                                              # null dk
    assert call(a12=rh.RehyatPhiGrad(4096, 4096, 0, 4096)) == 1          # null dW_k
    assert call(a4=rh.RehyatPhi(4096, 0, 4096, 4096)) == 1               # null b_q
    assert call(a9=4104) == 3                                            # dq not 16-byte aligned
    assert call(a7=4098) == 3                                            # c not 4-byte aligned
    assert call(a14=ws - 1) == 4
    assert call(a0=_params(flags=rh.FLAG_FP8_QK)) == 2
    assert call(a0=_params(D=48)) == 2
    assert rh.rehyat_hybrid_attn_bwd_workspace_bytes(_params(flags=rh.FLAG_FP8_QK)) == 0
    assert rh.rehyat_hybrid_attn_bwd_workspace_bytes(_params(T=0)) == 0
    # fp32 inputs or another D: no bf16 copy of dy / den.
    p32 = _params(in_dtype=rh.F32)
    assert (rh.rehyat_hybrid_attn_bwd_workspace_bytes(p32) - rh.rehyat_phi_bwd_workspace_bytes(p32)
            < 3 * 4 * rows + 3 * 256 + 1)


def test_denominator_report_needs_an_output():
    assert rh.lib().rehyat_denominator_report(None, 0) == 1


def test_header_is_plain_c_and_the_library_links_from_c(tmp_path):
    """include/rehyat.h compiles as strict C99 with no warnings, and a C
    program linked against librehyat.so gets the same answers as the
    binding (host-only calls; no GPU needed)."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    root = os.path.dirname(HEADER)
    pkg = os.path.dirname(rh.lib_path())
    src = tmp_path / "abi.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "abi"
    res = subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                          "-I" + root, str(src), "-L" + pkg, "-lrehyat",
                          "-Wl,-rpath," + pkg, "-o", str(exe)],
                         capture_output=True, text=True, timeout=120)
    assert res.returncode == 0, res.stderr
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stderr
    version, ws, path, st = (int(x) for x in out.stdout.split())
    p = rh.make_params(batch=2, heads=12, T=21, Hs=30, Ws=52, D=128, Dp=128, Tc=3, To=1,
                       causal=0)
    assert version == rh.rehyat_version()
    assert ws == rh.rehyat_workspace_bytes(p) > 0
    assert path == rh.rehyat_attn_path(p) == 1
    assert st == 1  # REHYAT_ERR_INVALID_ARG, before any launch


def test_step_key_split_choice():
    """The streaming step's key-window split: 0 for invalid arguments, 2
    pieces for 12 heads of 30x52 with T_c = 3, T_o = 1 on a 148-SM B200 (228
    CTAs would run in 1.54 waves; the pairs past the first wave split in two),
    none where the chunk already makes several waves or the CUDA-core path
    runs."""
    kw = dict(batch=1, heads=12, T=3, Hs=30, Ws=52, D=128, Dp=128, Tc=3, To=1, causal=1,
              in_dtype=rh.BF16, out_dtype=rh.F32)
    p = rh.make_params(**kw)
    assert rh.rehyat_step_key_split(p, 0) == 0
    assert rh.rehyat_step_key_split(p, 4) == 0
    assert rh.rehyat_step_key_split(p, 3) == 2
    assert rh.rehyat_step_key_split(rh.make_params(**{**kw, "batch": 8}), 3) == 1
    assert rh.rehyat_step_key_split(rh.make_params(**{**kw, "flags": rh.FLAG_FORCE_SIMT}), 3) == 1
    assert rh.rehyat_step_key_split(rh.make_params(**{**kw, "in_dtype": rh.F32}), 3) == 1
    # The workspace holds the partials of the split pairs: at most 12 x 19
    # pairs x 4 pieces x 2 tiles x 128 rows x 33 float4.
    ws = rh.rehyat_step_workspace_bytes(p)
    ws_simt = rh.rehyat_step_workspace_bytes(rh.make_params(**{**kw, "flags": rh.FLAG_FORCE_SIMT}))
    assert 0 < ws - ws_simt <= 12 * 19 * 4 * 2 * 128 * 33 * 16 + 256
