"""Host-side size logic of the C ABI (no GPU needed): workspace sizes of the
full forward, the fp8 variant and the host-buffer forward."""
import pytest

import linear_attention_video_chunked_b200 as rh

BASE = dict(batch=2, heads=12, T=21, Hs=30, Ws=52, D=128, Dp=128, Tc=3, To=1, causal=0)


def _lib_or_skip():
    try:
        rh.lib()
    except (OSError, RuntimeError) as e:  # library not built in this checkout
        pytest.skip(str(e))


def test_fp8_workspace_adds_the_two_e4m3_copies():
    _lib_or_skip()
    plain = rh.rehyat_workspace_bytes(rh.make_params(**BASE))
    fp8 = rh.rehyat_workspace_bytes(rh.make_params(**BASE, flags=rh.FLAG_FP8_QK))
    n = 2 * 12 * 21 * 30 * 52 * 128
    assert plain > 0 and 2 * n <= fp8 - plain <= 2 * n + 512  # two copies, 256-byte aligned


@pytest.mark.parametrize("bad", [dict(in_dtype=rh.F32), dict(Dp=256), dict(D=64)])
def test_fp8_refused_for_unsupported_shapes(bad):
    _lib_or_skip()
    p = rh.make_params(**{**BASE, **{k: v for k, v in bad.items() if k != "in_dtype"}},
                       in_dtype=bad.get("in_dtype", rh.BF16), flags=rh.FLAG_FP8_QK)
    assert rh.rehyat_workspace_bytes(p) == 0


def test_host_workspace_grows_with_the_slab_and_saturates():
    _lib_or_skip()
    p = rh.make_params(**BASE)
    sizes = [rh.rehyat_host_workspace_bytes(p, s) for s in (1, 2, 3, 4, 6, 12)]
    assert all(a < b for a, b in zip(sizes, sizes[1:]))
    # heads_per_slab <= 0 or >= heads: one slab per batch element.
    assert rh.rehyat_host_workspace_bytes(p, 0) == sizes[-1]
    assert rh.rehyat_host_workspace_bytes(p, 99) == sizes[-1]
    # Three slots of q, k, v (bf16) and y (fp32) for one slab, plus its forward.
    one = 21 * 30 * 52 * 128
    slab = rh.make_params(**{**BASE, "batch": 1, "heads": 2})
    want = 3 * 2 * one * (3 * 2 + 4) + rh.rehyat_workspace_bytes(slab)
    assert want <= sizes[1] <= want + 16 * 256
    # Invalid parameters: 0.
    assert rh.rehyat_host_workspace_bytes(rh.make_params(**{**BASE, "D": 48}), 2) == 0
