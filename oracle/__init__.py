"""fp64 CPU oracle for the sign-weight linear layers (OneBit and DBF).

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or link
this package: only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` use it.  It shares no code with the CUDA library (no common
helpers, tables or constants) and never takes an input or an expected value from
the CUDA path.

Everything is plain NumPy in float64, written from the definitions on the pages:

* OneBit, from "1bit量化" (blog.zerodtree.com, notes on "OneBit: Towards
  Extremely Low-bit Large Language Models"): sign/value split and rank-1 SVID
  (section "rank-1 approximation"), Proposition 1, Lemma 1, Proposition 2, and
  the LayerNorm that follows the layer (knowledge-distillation section).
* DBF, from "Addition is almost all you need: Compressing large language models
  with double binary factorization" (gist.science, section "Methodologie:
  Double Binary Factorization (DBF)"): the factorised weight and its inference
  chain; and, in the submodule ``oracle.dbf_factorize``, the factorisation
  W -> (S_A, S_B, a, m, b) by alternating ADMM steps with an SVID projection
  ("Optimalisatie en Training").

The linear layers are computed in the DIRECT form -- the approximated weight
matrix is materialised and then multiplied -- not in the factorised order the
kernels use, so that agreement is evidence rather than repetition.

Parity status: every public function of ``oracle.onebit`` and ``oracle.dbf`` is
pinned by tests under ``tests/test_oracle_*.py`` against hand-computed worked
examples (``tests/golden/``), closed forms, special cases and brute force.  In
``oracle.dbf_factorize`` the steps are pinned the same way (projection, ADMM
least-squares steps, scale refits), but the factorisation loop as a whole is
"parity unpinned": the page names a heuristic without giving its steps, so only
exact recovery and properties of the result can be checked.
"""
from .onebit import (sign_pm1, pack_signs, unpack_signs, rank1_svd, svid_rank1,
                     onebit_weight, onebit_linear, onebit_linear_packed,
                     onebit_linear_prop1, layernorm, onebit_linear_ln, LN_EPS)
from .dbf import dbf_weight, dbf_linear, dbf_linear_chain
from . import dbf_factorize

__all__ = [
    "sign_pm1", "pack_signs", "unpack_signs", "rank1_svd", "svid_rank1",
    "onebit_weight", "onebit_linear", "onebit_linear_packed", "onebit_linear_prop1",
    "layernorm", "onebit_linear_ln", "LN_EPS",
    "dbf_weight", "dbf_linear", "dbf_linear_chain", "dbf_factorize",
]
