"""Readers for the hand-derived fixtures under tests/golden/."""
import os
from fractions import Fraction

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _lines(name):
    with open(os.path.join(GOLDEN, name)) as fh:
        for ln in fh:
            ln = ln.strip()
            if ln and not ln.startswith("#"):
                yield ln


def capacity_cases():
    out = []
    for ln in _lines("capacity.txt"):
        T, N, cf, C = ln.split()
        out.append((int(T), int(N), float(cf), int(C)))
    return out


def softmax_cases():
    out = []
    for ln in _lines("softmax_hand.txt"):
        a, p, top = (s.strip() for s in ln.split("|"))
        out.append(([int(v) for v in a.split()],
                    [Fraction(v) for v in p.split()], int(top)))
    return out


def aux_loss_cases():
    out = []
    for ln in _lines("aux_loss_hand.txt"):
        name, groups, f, P, loss = (s.strip() for s in ln.split("|"))
        toks = []
        for g in groups.split():
            cnt, vals = g.split("x")
            toks += [[int(v) for v in vals.split(",")]] * int(cnt)
        out.append((name, toks, [Fraction(v) for v in f.split()],
                    [Fraction(v) for v in P.split()], float(loss)))
    return out


def dispatch_case():
    kv = {}
    for ln in _lines("dispatch_hand.txt"):
        k, *v = ln.split()
        kv[k] = [int(x) for x in v]
    return kv


def top2_router_cases():
    out = []
    for ln in _lines("top2_hand.txt"):
        if not ln.startswith("router"):
            continue
        a, g, top = (s.strip() for s in ln[len("router"):].split("|"))
        out.append(([int(v) for v in a.split(",")], [Fraction(v) for v in g.split()],
                    [int(v) for v in top.split()]))
    return out


def top2_dispatch_case():
    kv = {}
    for ln in _lines("top2_hand.txt"):
        if ln.startswith("router"):
            continue
        k, *v = ln.split()
        kv[k] = [int(x) for x in v]
    return kv
