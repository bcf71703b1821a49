"""The oracle's pins catch plausible mistakes planted in it.

Each case takes the oracle's source, plants one mistake by a text replacement (a
reversed bit order, a wrong sign threshold, a dropped |.|, the smallest instead of
the largest singular triple, a flipped unpack polarity, a dropped middle or input
scale, reversed columns, an unbiased variance, a missing mean subtraction),
executes the result as fresh in-memory
modules (nothing is written to disk) and runs a compact set of the pins against
it: the hand-worked fixtures under tests/golden/, the pack/unpack round trip,
Proposition 2's closed form and the DBF chain against the direct form.  Every
mutant must fail at least one pin; the unmodified oracle must pass all of them.
"""
import json
import os
import types

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
GOLDEN = os.path.join(ROOT, "tests", "golden")


def _load(mutation=None):
    """The oracle's public functions from its sources, with one optional (file, old, new) replacement.

    onebit.py and dbf.py import only numpy, so each executes on its own.
    """
    ns = types.SimpleNamespace()
    for fname in ("onebit.py", "dbf.py"):
        src = open(os.path.join(ROOT, "oracle", fname), encoding="utf-8").read()
        if mutation and mutation[0] == fname:
            assert mutation[1] in src, mutation
            src = src.replace(mutation[1], mutation[2], 1)
        mod = types.ModuleType("oracle_" + fname[:-3])
        exec(compile(src, "oracle/" + fname, "exec"), mod.__dict__)
        for k, v in vars(mod).items():
            if not k.startswith("_"):
                setattr(ns, k, v)
    return ns


def _golden(name):
    with open(os.path.join(GOLDEN, name), encoding="utf-8") as f:
        return json.load(f)


def _pins(o):
    """Run the pins; return the list of the ones that fail."""
    failed = []

    def check(name, fn):
        try:
            if not fn():
                failed.append(name)
        except Exception:  # a pin that raises has failed
            failed.append(name)

    def pack_golden():
        g = _golden("pack_words.json")
        rows, words = [], []
        for row in g["rows"]:
            r = np.full(g["K"], row["fill"], dtype=np.float32)
            for col, val in row["set"].items():
                r[int(col)] = np.float32(float(val))
            rows.append(r)
            words.append([int(w, 16) for w in row["words"]])
        return o.pack_signs(np.stack(rows)).tolist() == words

    def pack_roundtrip():
        W = np.random.default_rng(1).standard_normal((5, 96)).astype(np.float32)
        return np.array_equal(o.unpack_signs(o.pack_signs(W), 96), o.sign_pm1(W))

    def svid_golden():
        ok = True
        for name in ("svid_2x2.json", "svid_3x2_diag.json"):
            g = _golden(name)
            a, b, s = o.svid_rank1(np.array(g["W"]))
            ok &= abs(s - g["sigma1"]) < 1e-9
            ok &= np.allclose(a, g["a"], atol=1e-9) and np.allclose(b, g["b"], atol=1e-9)
            ok &= np.allclose(o.onebit_weight(o.sign_pm1(np.array(g["W"])), a, b), g["W_hat"], atol=1e-9)
        return ok

    def prop2_closed_form():
        W = np.random.default_rng(2).standard_normal((12, 9))
        a, b, s = o.svid_rank1(W)
        A = np.abs(W)
        return abs(np.linalg.norm(A - np.outer(a, b)) ** 2 - (np.linalg.norm(A) ** 2 - s ** 2)) < 1e-9

    def linear_golden():
        g = _golden("onebit_linear_2x2.json")
        return np.allclose(o.onebit_linear(np.array(g["X"]), np.array(g["S"]), np.array(g["a"]), np.array(g["b"])),
                           g["Y"], atol=1e-9)

    def dbf_golden():
        g = _golden("dbf_2x2.json")
        Y = o.dbf_linear(np.array(g["X"]), np.array(g["S_A"]), np.array(g["S_B"]), np.array(g["a"]),
                         np.array(g["m"]), np.array(g["b"]))
        return np.allclose(Y, g["Y"], atol=1e-9)

    def dbf_chain():
        rng = np.random.default_rng(3)
        SA, SB = np.sign(rng.standard_normal((6, 4))), np.sign(rng.standard_normal((4, 5)))
        a, m, b = rng.uniform(0.5, 2, 6), rng.uniform(0.5, 2, 4), rng.uniform(0.5, 2, 5)
        X = rng.standard_normal((3, 5))
        return np.allclose(o.dbf_linear(X, SA, SB, a, m, b), o.dbf_linear_chain(X, SA, SB, a, m, b), atol=1e-10)

    def layernorm_golden():
        g = _golden("layernorm_4.json")
        return np.allclose(o.layernorm(np.array(g["Y"]), eps=g["eps"]), g["Z"], atol=1e-12)

    for name, fn in (("pack_golden", pack_golden), ("pack_roundtrip", pack_roundtrip), ("svid_golden", svid_golden),
                     ("prop2_closed_form", prop2_closed_form), ("linear_golden", linear_golden),
                     ("dbf_golden", dbf_golden), ("dbf_chain", dbf_chain), ("layernorm_golden", layernorm_golden)):
        check(name, fn)
    return failed


MUTATIONS = [
    ("onebit.py", "<< np.uint64(i)", "<< np.uint64(31 - i)"),                                  # reversed bit order
    ("onebit.py", "np.where(W < 0, -1.0, 1.0)", "np.where(W <= 0, -1.0, 1.0)"),              # Sign(0) = -1
    ("onebit.py", "A = np.abs(np.asarray(W, dtype=np.float64))", "A = np.asarray(W, dtype=np.float64)"),  # no |W|
    ("onebit.py", "return U[:, 0].copy(), float(s[0]), Vt[0].copy()",
     "return U[:, -1].copy(), float(s[-1]), Vt[-1].copy()"),                                 # smallest triple
    ("onebit.py", "out[:, i::32] = np.where(bit == 1, -1.0, 1.0)",
     "out[:, i::32] = np.where(bit == 1, 1.0, -1.0)"),                                        # unpack polarity
    ("dbf.py", "left = a[:, None] * S_A * m[None, :]", "left = a[:, None] * S_A"),            # dropped m
    ("dbf.py", "right = S_B * b[None, :]", "right = S_B"),                                   # dropped b
    ("dbf.py", "return left @ right", "return left @ right[:, ::-1]"),                       # reversed columns
    ("onebit.py", "var = ((Y - mean) ** 2).mean(axis=1, keepdims=True)",
     "var = ((Y - mean) ** 2).sum(axis=1, keepdims=True) / (Y.shape[1] - 1)"),              # unbiased variance
    ("onebit.py", "return (Y - mean) / np.sqrt(var + eps)", "return Y / np.sqrt(var + eps)"),  # no mean removal
]


def test_unmodified_oracle_passes_the_pins():
    assert _pins(_load()) == []


@pytest.mark.parametrize("mutation", MUTATIONS, ids=[m[1][:40] for m in MUTATIONS])
def test_each_planted_mistake_fails_a_pin(mutation):
    assert _pins(_load(mutation)), f"mutation survived: {mutation}"
