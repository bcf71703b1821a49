"""The oracle's pins catch plausible mistakes planted in it.

Each case takes the oracle's source, plants one mistake by a text replacement (a
reversed bit order, a wrong sign threshold, a dropped |.|, the smallest instead of
the largest singular triple, a flipped unpack polarity, a dropped middle or input
scale, reversed columns, an unbiased variance, a missing mean subtraction; in the
factorisation a dropped ADMM penalty or pull, a wrong dual sign, dropped signs in
the projection, half of the middle scale lost, a matrix instead of a Hadamard
product in the Gram matrix, a biased refit, a mis-scaled start ridge), executes
the result as fresh in-memory modules (nothing is written to disk) and runs a
compact set of the pins against it: the hand-worked fixtures under tests/golden/,
the pack/unpack round trip, Proposition 2's closed form, the DBF chain against the
direct form, the projection's closed-form error, the ADMM steps and scale refits
against library least squares, the sketch start's closed form on a rank-1 weight,
exact recovery of a rank-1 DBF weight and the low-rank property.
Every mutant must fail at least one pin; the unmodified oracle must pass all of
them.
"""
import json
import os
import types

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
GOLDEN = os.path.join(ROOT, "tests", "golden")


# dbf_factorize.py takes these names from its sibling modules; the loader strips the
# relative imports and hands it the (possibly mutated) versions loaded before it.
_SIBLING_IMPORTS = "from .dbf import dbf_weight\nfrom .onebit import sign_pm1, svid_rank1\n"


def _load(mutation=None):
    """The oracle's public functions from its sources, with one optional (file, old, new) replacement.

    onebit.py and dbf.py import only numpy, so each executes on its own.
    """
    ns = types.SimpleNamespace()
    for fname in ("onebit.py", "dbf.py", "dbf_factorize.py"):
        src = open(os.path.join(ROOT, "oracle", fname), encoding="utf-8").read()
        if mutation and mutation[0] == fname:
            assert mutation[1] in src, mutation
            src = src.replace(mutation[1], mutation[2], 1)
        mod = types.ModuleType("oracle_" + fname[:-3])
        if fname == "dbf_factorize.py":
            assert _SIBLING_IMPORTS in src
            src = src.replace(_SIBLING_IMPORTS, "")
            mod.__dict__.update(dbf_weight=ns.dbf_weight, sign_pm1=ns.sign_pm1, svid_rank1=ns.svid_rank1)
        exec(compile(src, "oracle/" + fname, "exec"), mod.__dict__)
        for k, v in vars(mod).items():
            if not k.startswith("_") and not (fname == "dbf_factorize.py" and hasattr(ns, k)):
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

    def projection_closed_form():
        M = np.random.default_rng(4).standard_normal((7, 5))
        Z = o.structured(*o.svid_project(M))
        lam = np.linalg.eigvalsh(np.abs(M).T @ np.abs(M))[-1]
        return abs(np.linalg.norm(M - Z) ** 2 - (np.linalg.norm(M) ** 2 - lam)) < 1e-9

    def admm_step_lstsq():
        rng = np.random.default_rng(5)
        W, ZA, UA = rng.standard_normal((4, 7)), rng.standard_normal((4, 3)), rng.standard_normal((4, 3))
        ZB, UB = rng.standard_normal((3, 7)), rng.standard_normal((3, 7))
        rho = 0.6
        A = o.admm_left_step(W, ZB, ZA, UA, rho)
        DA = np.vstack([ZB.T, np.sqrt(rho) * np.eye(3)])
        ok = all(np.allclose(A[n], np.linalg.lstsq(DA, np.concatenate([W[n], np.sqrt(rho) * (ZA - UA)[n]]),
                                                    rcond=None)[0]) for n in range(4))
        B = o.admm_right_step(W, ZA, ZB, UB, rho)
        DB = np.vstack([ZA, np.sqrt(rho) * np.eye(3)])
        ok &= all(np.allclose(B[:, k], np.linalg.lstsq(DB, np.concatenate([W[:, k], np.sqrt(rho) * (ZB - UB)[:, k]]),
                                                        rcond=None)[0]) for k in range(7))
        return ok

    def refit_lstsq():
        rng = np.random.default_rng(6)
        W = rng.standard_normal((5, 6))
        SA, SB = np.sign(rng.standard_normal((5, 3))), np.sign(rng.standard_normal((3, 6)))
        a, m, b = rng.uniform(0.5, 2, 5), rng.uniform(0.5, 2, 3), rng.uniform(0.5, 2, 6)
        D = np.stack([np.outer(a * SA[:, j], SB[j] * b).ravel() for j in range(3)], axis=1)
        ok = np.allclose(o.refit_m(W, SA, SB, a, b), np.linalg.lstsq(D, W.ravel(), rcond=None)[0])
        R = SA @ np.diag(m) @ SB @ np.diag(b)
        ok &= np.allclose(o.refit_a(W, SA, SB, m, b), (W * R).sum(1) / (R * R).sum(1))
        C = np.diag(a) @ SA @ np.diag(m) @ SB
        ok &= np.allclose(o.refit_b(W, SA, SB, a, m), (W * C).sum(0) / (C * C).sum(0))
        return ok

    def factorize_exact_rank1():
        rng = np.random.default_rng(7)
        W = o.dbf_weight(np.sign(rng.standard_normal((6, 1))), np.sign(rng.standard_normal((1, 8))),
                         rng.uniform(0.2, 2, 6), rng.uniform(0.5, 2, 1), rng.uniform(0.2, 2, 8))
        res = o.dbf_factorize(W, 1, sweeps=2, refit_rounds=0)
        return res["error"] <= 1e-10 * np.linalg.norm(W)

    def sketch_start_closed_form():
        rng = np.random.default_rng(8)
        W = o.dbf_weight(np.sign(rng.standard_normal((6, 1))), np.sign(rng.standard_normal((1, 8))),
                         rng.uniform(0.2, 2, 6), rng.uniform(0.5, 2, 1), rng.uniform(0.2, 2, 8))
        A, B = o.dbf_init_sketch(W, rng.standard_normal((8, 4)))
        return np.allclose(A @ B, W / (1 + o.SKETCH_RIDGE / 4), rtol=1e-10, atol=1e-12)

    def factorize_low_rank():
        rng = np.random.default_rng(0)
        N, K = 96, 128
        W = rng.standard_normal((N, 8)) @ rng.standard_normal((8, K)) * 0.01 + 0.001 * rng.standard_normal((N, K))
        a, b, _ = o.svid_rank1(W)
        e1 = np.linalg.norm(W - o.onebit_weight(o.sign_pm1(W), a, b))
        return o.dbf_factorize(W, N * K // (N + K))["error"] < 0.6 * e1

    for name, fn in (("pack_golden", pack_golden), ("pack_roundtrip", pack_roundtrip), ("svid_golden", svid_golden),
                     ("prop2_closed_form", prop2_closed_form), ("linear_golden", linear_golden),
                     ("dbf_golden", dbf_golden), ("dbf_chain", dbf_chain), ("layernorm_golden", layernorm_golden),
                     ("projection_closed_form", projection_closed_form), ("admm_step_lstsq", admm_step_lstsq),
                     ("refit_lstsq", refit_lstsq), ("factorize_exact_rank1", factorize_exact_rank1),
                     ("sketch_start_closed_form", sketch_start_closed_form),
                     ("factorize_low_rank", factorize_low_rank)):
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
    ("dbf_factorize.py", "G = ZB @ ZB.T + rho * np.eye(r)", "G = ZB @ ZB.T"),                  # penalty dropped
    ("dbf_factorize.py", "R = W @ ZB.T + rho * (ZA - UA)", "R = W @ ZB.T + rho * (ZA + UA)"),  # dual sign
    ("dbf_factorize.py", "R = ZA.T @ W + rho * (ZB - UB)", "R = ZA.T @ W"),                   # right pull dropped
    ("dbf_factorize.py", "return sign_pm1(M), u, v", "return sign_pm1(np.abs(M)), u, v"),      # signs dropped
    ("dbf_factorize.py", "a, m, b = uA, vA * uB, vB", "a, m, b = uA, vA, vB"),                 # middle scale half lost
    ("dbf_factorize.py", "G = (P.T @ P) * (Q @ Q.T)", "G = (P.T @ P) @ (Q @ Q.T)"),             # Gram product
    ("dbf_factorize.py", "den = (C * C).sum(axis=0)", "den = (C * C).sum(axis=0) + 1.0"),      # biased b refit
    ("dbf_factorize.py", "eps = SKETCH_RIDGE * float(np.trace(G)) / r", "eps = SKETCH_RIDGE * float(np.trace(G))"),
]


def test_unmodified_oracle_passes_the_pins():
    assert _pins(_load()) == []


@pytest.mark.parametrize("mutation", MUTATIONS, ids=[m[1][:40] for m in MUTATIONS])
def test_each_planted_mistake_fails_a_pin(mutation):
    assert _pins(_load(mutation)), f"mutation survived: {mutation}"
