"""Write the exact-rational fixtures in this folder.  Calls only ``oracle/``.

The pages print no worked numeric example, so the fixtures are tiny cases whose
expected values are computed in exact rational arithmetic by the transition-
matrix brute force in ``oracle/exact.py`` (per-token update of
"NVIDIA AIがGated DeltaNet-2を発表", ai.warp-studio.com, section
"Gated DeltaNet-2の核心"; special cases from "Jerarquía de Generalización",
needhelp.icu).  All inputs are dyadic rationals, so they are exact in fp64.

Run from the repository root:  python tests/golden/make_golden.py
"""
import json
import os
import sys
from fractions import Fraction as F

sys.path.insert(0, os.path.abspath(os.path.join(os.path.dirname(__file__), "..", "..")))
from oracle import exact  # noqa: E402

HERE = os.path.dirname(os.path.abspath(__file__))


def s(x):
    return str(x)


def dump(name, cite, inputs, outs, ST, extra=None):
    doc = {"citation": cite, "inputs": {k: [[s(x) for x in row] for row in v] if isinstance(v[0], list) else [s(x) for x in v]
                                         for k, v in inputs.items()},
           "o": [[s(x) for x in row] for row in outs], "S_T": [[s(x) for x in row] for row in ST]}
    if extra:
        doc.update(extra)
    with open(os.path.join(HERE, name), "w") as f:
        json.dump(doc, f, indent=1)
        f.write("\n")


def main():
    # GDN-2, T=3, d_k=2, d_v=3, nonzero S0
    q = [[F(1, 2), F(-1, 4)], [F(3, 4), F(1, 8)], [F(-1, 2), F(1, 2)]]
    k = [[F(1, 2), F(1, 2)], [F(-3, 4), F(1, 4)], [F(1, 8), F(-7, 8)]]
    v = [[F(1), F(-1, 2), F(1, 4)], [F(-3, 8), F(5, 8), F(1, 2)], [F(1, 4), F(1, 4), F(-1)]]
    alpha = [[F(1, 2), F(7, 8)], [F(3, 4), F(1)], [F(15, 16), F(1, 4)]]
    b = [[F(1, 4), F(3, 4)], [F(1, 2), F(1, 8)], [F(7, 8), F(1, 2)]]
    w = [[F(3, 4), F(1, 2), F(1, 8)], [F(1, 4), F(7, 8), F(1, 2)], [F(1, 2), F(5, 8), F(3, 8)]]
    S0 = [[F(1, 16), F(-1, 8), F(0)], [F(1, 4), F(1, 32), F(-1, 16)]]
    outs, ST = exact.gdn2_transition_products(q, k, v, alpha, b, w, S0)
    dump("gdn2_tiny_exact.json",
         "Gated Delta Rule-2 per-token update: decay first, key-side erase gate b, value-side "
         "write gate w, o_t = S_t^T q_t ('NVIDIA AIがGated DeltaNet-2を発表', ai.warp-studio.com, "
         "'Gated DeltaNet-2の核心'); erase reading k (b*k)^T; exact rational transition-matrix brute force",
         dict(q=q, k=k, v=v, alpha=alpha, b=b, w=w, S0=S0), outs, ST)

    # KDA special case: the GDN-2 inputs above with b = w = beta (scalar per token)
    beta = [F(1, 2), F(3, 4), F(1, 4)]
    outs, ST = exact.kda_textbook(q, k, v, alpha, beta, S0)
    dump("kda_tiny_exact.json",
         "KDA = GDN-2 when b_t and w_t collapse to one scalar ('Jerarquía de Generalización', "
         "needhelp.icu; 'Gated DeltaNet-2の核心', ai.warp-studio.com); expected values from the textbook "
         "KDA recurrence S = (I - beta k k^T) Diag(alpha) S + beta k v^T in exact rationals",
         dict(q=q, k=k, v=v, alpha=alpha, S0=S0, beta=beta), outs, ST)

    # Gated DeltaNet special case: alpha also scalar per token
    a_s = [F(1, 2), F(7, 8), F(3, 4)]
    outs, ST = exact.gdn_textbook(q, k, v, a_s, beta, S0)
    dump("gdn_tiny_exact.json",
         "Gated DeltaNet = KDA when the per-channel decay collapses to a scalar ('Jerarquía de "
         "Generalización', needhelp.icu); expected values from the textbook Gated DeltaNet recurrence "
         "S = alpha (I - beta k k^T) S + beta k v^T in exact rationals",
         dict(q=q, k=k, v=v, S0=S0, beta=beta, alpha_scalar=a_s), outs, ST)


if __name__ == "__main__":
    main()
