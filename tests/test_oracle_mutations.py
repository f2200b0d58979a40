"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in an in-memory copy of an oracle module (a
dropped term, a wrong sign, index or operand, an off-by-one window, the
other reading of an ambiguous step), points that module's pin tests at the
copy, and runs them on the CPU: at least one must fail.  A control run of
the unmodified copy through the same harness must pass, so a failure is the
planted mistake's doing.  The files under oracle/ are never modified.
"""
import importlib
import inspect
import itertools
import os
import types

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# oracle module -> its pin tests
PINS = {
    "oracle.rehyat_oracle": "tests.test_oracle",
    "oracle.rehyat_phi_grad": "tests.test_phi_grad_oracle",
    "oracle.rehyat_grad": "tests.test_grad_oracle",
    "oracle.rehyat_phi_mlp": "tests.test_phi_mlp_oracle",
    "oracle.rehyat_fp8": "tests.test_fp8_oracle",
}

# (module, planted mistake, text in the module (exactly once), replacement)
MUTANTS = [
    # Feature map (Key design 3).
    ("oracle.rehyat_oracle", "phi: first part not squared",
     "[psi_1 ** 2, psi_2 ** 2]", "[psi_1, psi_2 ** 2]"),
    ("oracle.rehyat_oracle", "phi: second part takes the first bias",
     "psi_2 = x @ W[1] + b[1]", "psi_2 = x @ W[1] + b[0]"),
    ("oracle.rehyat_oracle", "phi: bias subtracted",
     "psi_1 = x @ W[0] + b[0]", "psi_1 = x @ W[0] - b[0]"),
    # Chunks and windows (Key designs 1 and 2).
    ("oracle.rehyat_oracle", "window one overlap slice short",
     "rows.append((first, end, max(first - To, 0)))",
     "rows.append((first, end, max(first - max(To - 1, 0), 0)))"),
    ("oracle.rehyat_oracle", "ragged last chunk not clipped at T",
     "end = min(T, first + Tc)", "end = first + Tc"),
    ("oracle.rehyat_oracle", "pairwise: overlap counted in tokens, not slices",
     "lo = max(t * Np - To * HW, 0)", "lo = max(t * Np - To, 0)"),
    ("oracle.rehyat_oracle", "pairwise: bidirectional linear set loses the keys before the window",
     "lin = (j < lo) if causal else ~soft", "lin = (j < lo) if causal else (j >= hi)"),
    ("oracle.rehyat_oracle", "pairwise: stabiliser over all keys, not the window",
     "c = logits[soft].max()", "c = logits.max()"),
    ("oracle.rehyat_oracle", "pairwise: phi_q and phi_k swapped in the linear weight",
     "w_lin = np.where(lin, fk @ fq[i], 0.0)", "w_lin = np.where(lin, fq @ fk[i], 0.0)"),
    # Factored form.
    ("oracle.rehyat_oracle", "factored: logits not scaled",
     "logits = (ql[rows] @ kl[start * HW:end * HW].T) * scale",
     "logits = (ql[rows] @ kl[start * HW:end * HW].T)"),
    ("oracle.rehyat_oracle", "factored: S_L built from keys instead of values",
     "S_L = fk.T @ v[lin]", "S_L = fk.T @ k[lin]"),
    ("oracle.rehyat_oracle", "factored: bidirectional linear set loses the keys after the chunk",
     "lin = before if causal else np.concatenate([before, after])", "lin = before"),
    ("oracle.rehyat_oracle", "factored: n^L dropped from the denominator",
     "y[rows] = (aS + aL) / (nS + nL)[:, None]", "y[rows] = (aS + aL) / nS[:, None]"),
    ("oracle.rehyat_oracle", "factored: phi_q evaluated with phi_k's parameters",
     "fq = feature_map(Qc, Wq, bq)", "fq = feature_map(Qc, Wk, bk)"),
    ("oracle.rehyat_oracle", "scale 1/D instead of 1/sqrt(D)",
     "return 1.0 / math.sqrt(D) if scale is None", "return 1.0 / D if scale is None"),
    # Chunk-wise RNN (Key design 4).
    ("oracle.rehyat_oracle", "rnn: the whole softmax window folded into the state "
                             "(the printed update, which counts the overlap twice)",
     "fk = feature_map(Kw[:leave * HW], self.Wk, self.bk)\n"
     "        self.s = self.s + fk.T @ Vw[:leave * HW]",
     "fk = feature_map(Kw, self.Wk, self.bk)\n"
     "        self.s = self.s + fk.T @ Vw"),
    ("oracle.rehyat_oracle", "rnn: z not updated",
     "self.z = self.z + fk.sum(axis=0)", "self.z = self.z"),
    ("oracle.rehyat_oracle", "rnn: ring keeps T_o slices before that many were seen",
     "keep = min(self.To, self.seen)", "keep = self.To"),
    # Gradient of the feature-map parameters.
    ("oracle.rehyat_phi_grad", "dphi_q: sign of the z_L term",
     "dfq[rows] += e @ S_L.T - r[:, None] * z_L[None, :]",
     "dfq[rows] += e @ S_L.T + r[:, None] * z_L[None, :]"),
    ("oracle.rehyat_phi_grad", "dphi_k: h_t dropped",
     "dfk[lin] += v[lin] @ G.T + h[None, :]", "dfk[lin] += v[lin] @ G.T"),
    ("oracle.rehyat_phi_grad", "du: factor 2 of the square dropped",
     "duq = 2.0 * uq[p] * dfq[:, cols]", "duq = uq[p] * dfq[:, cols]"),
    ("oracle.rehyat_phi_grad", "dW_k from q",
     "dWk[p] = k.T @ duk", "dWk[p] = q.T @ duk"),
    ("oracle.rehyat_phi_grad", "G_t from g instead of g / den",
     "G = fq[rows].T @ e", "G = fq[rows].T @ g"),
    ("oracle.rehyat_phi_grad", "causal linear set includes later keys",
     "lin = before if causal else np.concatenate([before, after])",
     "lin = np.concatenate([before, after])"),
    ("oracle.rehyat_phi_grad", "db_k from the query side",
     "dbk[p] = duk.sum(axis=0)", "dbk[p] = duq.sum(axis=0)"),
    # Full backward (gradients of q, k, v and the feature-map parameters).
    ("oracle.rehyat_grad", "backward: gradient through the maximum c dropped",
     "dS[np.arange(dS.shape[0]), jmax] -= Dc", "dS[np.arange(dS.shape[0]), jmax] -= 0.0"),
    ("oracle.rehyat_grad", "backward: gradient through the maximum with the wrong sign",
     "dS[np.arange(dS.shape[0]), jmax] -= Dc", "dS[np.arange(dS.shape[0]), jmax] += Dc"),
    ("oracle.rehyat_grad", "backward: maximum's gradient without the n^S term",
     "Dc = (gh * aS).sum(axis=1) - r * nS", "Dc = (gh * aS).sum(axis=1)"),
    ("oracle.rehyat_grad", "backward: denominator term with the wrong sign",
     "dE = gh @ v[win].T - r[:, None]", "dE = gh @ v[win].T + r[:, None]"),
    ("oracle.rehyat_grad", "backward: dk without the logit scale",
     "dk[win] += scale * (dS.T @ q[rows])", "dk[win] += dS.T @ q[rows]"),
    ("oracle.rehyat_grad", "backward: dq from the values",
     "dq[rows] += scale * (dS @ k[win])", "dq[rows] += scale * (dS @ v[win])"),
    ("oracle.rehyat_grad", "backward: softmax dv from g, not g / den",
     "dv[win] += E.T @ gh", "dv[win] += E.T @ g"),
    ("oracle.rehyat_grad", "backward: linear-branch dv dropped",
     "dv[lin] += fk[lin] @ G", "dv[lin] += 0.0 * fk[lin] @ G"),
    ("oracle.rehyat_grad", "backward: dq through phi_q dropped",
     'out["dq"] += duq @ Wq[p].T', 'out["dq"] += 0.0 * duq @ Wq[p].T'),
    ("oracle.rehyat_grad", "backward: dk through phi_k with W_q",
     'out["dk"] += duk @ Wk[p].T', 'out["dk"] += duk @ Wq[p].T'),
    ("oracle.rehyat_grad", "backward: window one overlap slice short (dk, dv of the overlap)",
     "win = slice(start * HW, end * HW)\n        lin = np.arange(0, start * HW) if causal else \\\n"
     "            np.concatenate([np.arange(0, start * HW), np.arange(end * HW, N)])\n"
     "        # Forward of this chunk.",
     "win = slice(min(start + 1, first) * HW, end * HW)\n        lin = np.arange(0, start * HW) if causal else \\\n"
     "            np.concatenate([np.arange(0, start * HW), np.arange(end * HW, N)])\n"
     "        # Forward of this chunk."),
    # General feature map and the phi-given forward.
    ("oracle.rehyat_phi_mlp", "GELU: erf argument not divided by sqrt(2)",
     "erf(x / math.sqrt(2.0))", "erf(x)"),
    ("oracle.rehyat_phi_mlp", "part i raised to the power i + 2",
     "** (i + 1) for i in range(P)", "** (i + 2) for i in range(P)"),
    ("oracle.rehyat_phi_mlp", "b_b dropped",
     "psi = psi @ np.asarray(Wb, np.float64) + np.asarray(bb, np.float64)",
     "psi = psi @ np.asarray(Wb, np.float64)"),
    ("oracle.rehyat_phi_mlp", "phi-given: causal linear set includes later keys",
     "lin = before if causal else np.concatenate([before, after])",
     "lin = np.concatenate([before, after])"),
    ("oracle.rehyat_phi_mlp", "phi-given: n^L dropped from the denominator",
     "y[rows] = (aS + aL) / (nS + nL)[:, None]", "y[rows] = (aS + aL) / nS[:, None]"),
    ("oracle.rehyat_phi_mlp", "phi-given: S_L from phi_q",
     "S_L = fk[lin].T @ v[lin]", "S_L = fq[lin].T @ v[lin]"),
    # E4M3 rounding and the fp8 softmax variant.
    ("oracle.rehyat_fp8", "E4M3 with two fraction bits",
     "E4M3_FRACTION_BITS = 3", "E4M3_FRACTION_BITS = 2"),
    ("oracle.rehyat_fp8", "E4M3 without saturation",
     "r = np.minimum(r, E4M3_MAX)", "r = r"),
    ("oracle.rehyat_fp8", "E4M3 subnormal spacing from 2^-7",
     "E4M3_MIN_NORMAL_EXP = -6", "E4M3_MIN_NORMAL_EXP = -7"),
    ("oracle.rehyat_fp8", "E4M3 ties rounded away from zero",
     "r = np.round(a / spacing) * spacing", "r = np.floor(a / spacing + 0.5) * spacing"),
    ("oracle.rehyat_fp8", "fp8 logits from an unrounded q",
     "q8, k8 = e4m3_round(q), e4m3_round(k)", "q8, k8 = q, e4m3_round(k)"),
    ("oracle.rehyat_fp8", "fp8: phi_q sees the rounded q",
     "_factored_head(q[b, h], k[b, h], v[b, h]", "_factored_head(q8[b, h], k[b, h], v[b, h]"),
]

_PARAM_SET = type(pytest.param(0))
_SKIPPED = pytest.skip.Exception


def _load(module, old=None, new=None):
    """A fresh copy of ``module`` built from its source, with ``old``
    replaced by ``new``."""
    path = os.path.join(ROOT, *module.split(".")) + ".py"
    src = open(path).read()
    if old is not None:
        assert src.count(old) == 1, f"{module}: the text to replace must occur once: {old!r}"
        src = src.replace(old, new)
    mod = types.ModuleType(module)
    mod.__file__ = path
    exec(compile(src, path, "exec"), mod.__dict__)
    return mod


def _calls(fn):
    """Keyword arguments of every parametrised case of a test function."""
    grids = []
    for mark in getattr(fn, "pytestmark", []):
        if mark.name != "parametrize":
            continue
        names = mark.args[0]
        names = [n.strip() for n in names.split(",")] if isinstance(names, str) else list(names)
        rows = []
        for val in mark.args[1]:
            vals = val.values if isinstance(val, _PARAM_SET) else (
                (val,) if len(names) == 1 else val)
            rows.append(dict(zip(names, vals)))
        grids.append(rows)
    for combo in itertools.product(*grids):
        kw = {}
        for d in combo:
            kw.update(d)
        yield kw


def _run_pins(monkeypatch, module, copy):
    """Run the pin tests of ``module`` against ``copy``.  Returns (number
    of cases run, first failing case or None)."""
    original = importlib.import_module(module)
    tests = importlib.import_module(PINS[module])
    for name, obj in list(vars(tests).items()):
        if obj is original:
            monkeypatch.setattr(tests, name, copy)
        elif getattr(obj, "__module__", None) == module and hasattr(copy, name):
            monkeypatch.setattr(tests, name, getattr(copy, name))
    fns = [f for n, f in vars(tests).items() if n.startswith("test_") and callable(f)]
    fns.sort(key=lambda f: inspect.getsourcelines(f)[1])
    ran = 0
    for fn in fns:
        for kw in _calls(fn):
            ran += 1
            try:
                fn(**kw)
            except _SKIPPED:
                continue
            except Exception as e:  # noqa: BLE001 -- any failure is a caught mistake
                return ran, f"{fn.__name__}({kw}): {type(e).__name__}"
    return ran, None


@pytest.mark.parametrize("module", sorted(PINS))
def test_unmodified_copy_passes_its_pins(monkeypatch, module):
    ran, failed = _run_pins(monkeypatch, module, _load(module))
    assert failed is None, failed
    assert ran >= 5


@pytest.mark.parametrize("module,what,old,new", MUTANTS, ids=[m[1] for m in MUTANTS])
def test_pins_catch_planted_mistake(monkeypatch, module, what, old, new):
    ran, failed = _run_pins(monkeypatch, module, _load(module, old, new))
    assert failed is not None, f"no pin of {module} caught: {what} ({ran} cases ran)"
