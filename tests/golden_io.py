"""Readers for the exact fixtures under tests/golden/ (rationals, bf16 bits)."""
from __future__ import annotations

import os
from fractions import Fraction

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _vec(s: str) -> list[Fraction]:
    return [Fraction(t.strip()) for t in s.split(",")]


def read_lines(name: str) -> list[list[str]]:
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            rows.append([t.strip() for t in line.split("|")])
    return rows


def wn_cases():
    """(w, g, rho, eps, gy, weff, grad_w, grad_g, renorm) as Fractions."""
    out = []
    for f in read_lines("wn_exact.txt"):
        w, g, rho, eps, gy, weff, gw, gg, rn = f
        out.append(dict(w=_vec(w), g=Fraction(g), rho=Fraction(rho), eps=Fraction(eps), gy=_vec(gy),
                        weff=_vec(weff), grad_w=_vec(gw), grad_g=Fraction(gg), renorm=_vec(rn)))
    return out


def act_cases():
    """(op, x, r|None, alpha|None, eps, expected bits)."""
    out = []
    for f in read_lines("l2_exact.txt"):
        op, x, r, a, eps, bits = f
        out.append(dict(op=op, x=_vec(x), r=None if r == "-" else _vec(r), alpha=None if a == "-" else _vec(a),
                        eps=Fraction(eps), bits=[int(b, 16) for b in bits.split(",")]))
    return out


def optim_cases():
    """(w, eps, rho, G, projected G, renormed w) as Fractions."""
    out = []
    for f in read_lines("optim_exact.txt"):
        w, eps, rho, G, P, rn = f
        out.append(dict(w=_vec(w), eps=Fraction(eps), rho=Fraction(rho), G=_vec(G), P=_vec(P), renorm=_vec(rn)))
    return out
