"""Each plausible slip planted in a copy of the oracle source must make at
least one pin of tests/test_oracle_pins.py (forward),
tests/test_oracle_backward_pins.py (backward) or tests/test_oracle_sasa_pins.py
(SASA) fail.  The copies are compiled on
the CPU into a temporary directory; the committed oracle is never changed."""
import inspect

import pytest

import oracle
from oracle import na2d_oracle as ora
from tests import test_oracle_backward_pins as bwd_pins
from tests import test_oracle_pins as pins
from tests import test_oracle_block_pins as block_pins
from tests import test_oracle_nd_pins as nd_pins
from tests import test_oracle_sasa_pins as sasa_pins

MUTATIONS = {
    "bias dropped": ("A[a * ks + c] = dot + bias_at(rpb, h, ks, r - i, t - j);",
                     "A[a * ks + c] = dot;"),
    "bias not divided by sqrt(d)": ("A[a * ks + c] = dot + bias_at(rpb, h, ks, r - i, t - j);",
                                    "A[a * ks + c] = dot + sqrt((double)d) * bias_at(rpb, h, ks, r - i, t - j);"),
    "bias rows and columns swapped": ("bias_at(rpb, h, ks, r - i, t - j)", "bias_at(rpb, h, ks, t - j, r - i)"),
    "bias displacement sign flipped": ("bias_at(rpb, h, ks, r - i, t - j)", "bias_at(rpb, h, ks, i - r, j - t)"),
    "window shifted by one": ("long s = i - ks / 2;", "long s = i - ks / 2 - 1;"),
    "window clamped one short": ("if (s > L - ks) s = L - ks;", "if (s > L - ks) s = L - ks - (L > ks);"),
    "keys used as values": ("weighted_sum_one(A, v,", "weighted_sum_one(A, k,"),
    "no max subtraction": ("A[t] = exp(scale * A[t] - m);", "A[t] = exp(scale * A[t]);"),
    "scale 1/d instead of 1/sqrt(d)": ("double scale = 1.0 / sqrt((double)d);\n#pragma omp parallel num_threads(threads_for(nthreads))\n    {\n        double *A = (double *)malloc(sizeof(double) * (size_t)ks * ks);\n#pragma omp for schedule(dynamic)\n        for (long row",
                                       "double scale = 1.0 / (double)d;\n#pragma omp parallel num_threads(threads_for(nthreads))\n    {\n        double *A = (double *)malloc(sizeof(double) * (size_t)ks * ks);\n#pragma omp for schedule(dynamic)\n        for (long row"),
    "window entries column-major": ("long r = si + a, t = sj + c;\n            const double *kv",
                                    "long r = si + c, t = sj + a;\n            const double *kv"),
    "column window sized by H": ("long sj = na2d_oracle_window_start(j, W, ks);\n    for (long a = 0; a < ks; a++) {\n        for (long c = 0; c < ks; c++) {\n            long r",
                                 "long sj = na2d_oracle_window_start(j < H ? j : H - 1, H, ks);\n    for (long a = 0; a < ks; a++) {\n        for (long c = 0; c < ks; c++) {\n            long r"),
}


# Slips in the backward pass, each checked against the backward pins.
BACKWARD_MUTATIONS = {
    "softmax Jacobian without the row term": ("double dA = P[n] * (dP[n] - pdp) * scale;",
                                               "double dA = P[n] * dP[n] * scale;"),
    "logit gradient not divided by sqrt(d)": ("double dA = P[n] * (dP[n] - pdp) * scale;",
                                              "double dA = P[n] * (dP[n] - pdp);"),
    "dk takes the key instead of the query": ("dk[ki + x] += dA * q[qi + x];", "dk[ki + x] += dA * k[ki + x];"),
    "dv weighted by dP instead of P": ("dv[ki + x] += P[n] * dout[qi + x];", "dv[ki + x] += dP[n] * dout[qi + x];"),
    "dq scattered to the key": ("dq[qi + x] += dA * k[ki + x];", "dq[ki + x] += dA * k[ki + x];"),
    "bias gradient at the transposed displacement": (
        "(si + a - i + ks - 1)) * span + (sj + c - j + ks - 1)] += dA;",
        "(sj + c - j + ks - 1)) * span + (si + a - i + ks - 1)] += dA;"),
    "dP from the query's own value": ("for (long x = 0; x < d; x++) s += dout[qi + x] * v[ki + x];",
                                      "for (long x = 0; x < d; x++) s += dout[qi + x] * v[qi + x];"),
}


# Slips in SASA, each checked against the SASA pins.
SASA_MUTATIONS = {
    "window clamped like NA": ("long r = i - half + a, t = j - half + c;\n                        double dot = 0.0;",
                               "long r = na2d_oracle_window_start(i, H, ks) + a, t = na2d_oracle_window_start(j, W, ks) + c;\n                        double dot = 0.0;"),
    "padding left out of the softmax": ("                        A[a * ks + c] = dot + bias;",
                                        "                        A[a * ks + c] = (r >= 0 && r < H && t >= 0 && t < W) ? dot + bias : -INFINITY;"),
    "no bias on the padding": ("                        A[a * ks + c] = dot + bias;",
                               "                        A[a * ks + c] = (r >= 0 && r < H && t >= 0 && t < W) ? dot + bias : 0.0;"),
    "bias index off by one": ("(a - half + ks - 1)) * span + (c - half + ks - 1)]", "(a - half + ks)) * span + (c - half + ks - 2)]"),
}


def _pin_cases(module=pins):
    """(name, callable) for every pin, with parametrized pins at each of their cases."""
    cases = []
    for name, fn in inspect.getmembers(module, inspect.isfunction):
        if not name.startswith("test_"):
            continue
        marks = getattr(fn, "pytestmark", [])
        params = [m for m in marks if m.name == "parametrize"]
        if not params:
            cases.append((name, fn, {}))
            continue
        argnames, values = params[0].args
        argnames = [a.strip() for a in argnames.split(",")] if isinstance(argnames, str) else list(argnames)
        for val in values:
            val = val if isinstance(val, tuple) else (val,)
            cases.append((name, fn, dict(zip(argnames, val))))
    return cases


@pytest.mark.parametrize("mutation", sorted(MUTATIONS))
def test_planted_mistake_is_caught(mutation, tmp_path):
    old, new = MUTATIONS[mutation]
    text = ora.source_text()
    assert text.count(old) >= 1, f"mutation anchor not found: {mutation}"
    lib = ora.compile_variant(text.replace(old, new), str(tmp_path / "mutant.so"))
    failed = []
    with ora.swapped_library(lib):
        for name, fn, kwargs in _pin_cases():
            try:
                fn(**kwargs)
            except Exception:  # an assertion, or an error a pin provokes
                failed.append(name)
    assert failed, f"no pin caught the planted mistake: {mutation}"


@pytest.mark.parametrize("mutation", sorted(BACKWARD_MUTATIONS))
def test_planted_backward_mistake_is_caught(mutation, tmp_path):
    old, new = BACKWARD_MUTATIONS[mutation]
    text = ora.source_text()
    assert text.count(old) == 1, f"mutation anchor not found once: {mutation}"
    lib = ora.compile_variant(text.replace(old, new), str(tmp_path / "mutant.so"))
    failed = []
    with ora.swapped_library(lib):
        for name, fn, kwargs in _pin_cases(bwd_pins):
            try:
                fn(**kwargs)
            except Exception:  # an assertion, or an error a pin provokes
                failed.append(name)
    assert failed, f"no pin caught the planted mistake: {mutation}"


@pytest.mark.parametrize("mutation", sorted(SASA_MUTATIONS))
def test_planted_sasa_mistake_is_caught(mutation, tmp_path):
    old, new = SASA_MUTATIONS[mutation]
    text = ora.source_text()
    assert text.count(old) == 1, f"mutation anchor not found once: {mutation}"
    lib = ora.compile_variant(text.replace(old, new), str(tmp_path / "mutant.so"))
    failed = []
    with ora.swapped_library(lib):
        for name, fn, kwargs in _pin_cases(sasa_pins):
            try:
                fn(**kwargs)
            except Exception:  # an assertion, or an error a pin provokes
                failed.append(name)
    assert failed, f"no pin caught the planted mistake: {mutation}"


# Slips in the NA block (a Python function of the oracle), each checked
# against the block pins.
BLOCK_MUTATIONS = {
    "q and k swapped in the split": ("q, k, v = (np.ascontiguousarray(qkv[:, :, :, s]",
                                     "k, q, v = (np.ascontiguousarray(qkv[:, :, :, s]"),
    "heads and channels swapped in the split": ("qkv = _round_to(qkv, store).reshape(B, H, W, 3, heads, dh)",
                                                "qkv = _round_to(qkv, store).reshape(B, H, W, 3, dh, heads).swapaxes(4, 5)"),
    "output bias dropped": ("        y = y + bo\n", "        y = y\n"),
    "heads concatenated in the wrong order": ("y = o.transpose(0, 2, 3, 1, 4).reshape(-1, C) @ wo",
                                              "y = o[:, ::-1].transpose(0, 2, 3, 1, 4).reshape(-1, C) @ wo"),
}


@pytest.mark.parametrize("mutation", sorted(BLOCK_MUTATIONS))
def test_planted_block_mistake_is_caught(mutation, monkeypatch):
    import textwrap

    old, new = BLOCK_MUTATIONS[mutation]
    src = textwrap.dedent(inspect.getsource(ora.block_forward))
    assert src.count(old) == 1, f"mutation anchor not found once: {mutation}"
    scope = dict(vars(ora))
    exec(compile(src.replace(old, new), "<mutant>", "exec"), scope)
    monkeypatch.setattr(oracle, "block_forward", scope["block_forward"])
    failed = []
    for name, fn, kwargs in _pin_cases(block_pins):
        try:
            fn(**kwargs)
        except Exception:  # an assertion, or an error a pin provokes
            failed.append(name)
    assert failed, f"no pin caught the planted mistake: {mutation}"


# Slips in NA over 1-3 axes with dilation, each checked against its pins.
ND_MUTATIONS = {
    "dilation ignored in the key positions": (
        "long j0 = r0 + (st0 + a) * dl0, j1 = r1 + (st1 + b) * dl1, j2 = r2 + (st2 + c) * dl2;",
        "long j0 = r0 + (st0 + a), j1 = r1 + (st1 + b), j2 = r2 + (st2 + c);"),
    "sub-grid length rounded down": ("long rr = i % dl, ii = i / dl, Lp = (L - rr + dl - 1) / dl;",
                                     "long rr = i % dl, ii = i / dl, Lp = L / dl;"),
    "bias as if every window were centred": ("(st1 + b - p1 + k1 - 1)) * s2",
                                             "(b + k1 / 2)) * s2"),
    "window not clamped": ("    if (s > Lp - ka) s = Lp - ka;\n    *r = rr;", "    *r = rr;"),
    "axes 1 and 2 swapped in the bias": ("(st1 + b - p1 + k1 - 1)) * s2 + (st2 + c - p2 + k2 - 1)]",
                                         "(st2 + c - p2 + k2 - 1)) * s2 + (st1 + b - p1 + k1 - 1)]"),
}


@pytest.mark.parametrize("mutation", sorted(ND_MUTATIONS))
def test_planted_nd_mistake_is_caught(mutation, tmp_path):
    old, new = ND_MUTATIONS[mutation]
    text = ora.source_text()
    assert text.count(old) == 1, f"mutation anchor not found once: {mutation}"
    lib = ora.compile_variant(text.replace(old, new), str(tmp_path / "mutant.so"))
    failed = []
    with ora.swapped_library(lib):
        for name, fn, kwargs in _pin_cases(nd_pins):
            try:
                fn(**kwargs)
            except Exception:  # an assertion, or an error a pin provokes
                failed.append(name)
    assert failed, f"no pin caught the planted mistake: {mutation}"
