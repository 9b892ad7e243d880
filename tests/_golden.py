"""Readers for the hand-worked fixtures under tests/golden/."""
import os

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                yield line


def layout_cases():
    cases, cur = [], None
    for line in _lines("layout_hand.txt"):
        if line.startswith("case"):
            T, k, E, R = map(int, line.split()[1:])
            cur = dict(T=T, k=k, E=E, R=R)
            cases.append(cur)
        else:
            key, vals = line.split(":", 1)
            cur[key.strip()] = [int(v) for v in vals.split()]
    return cases


def e4m3_codes():
    out = []
    for line in _lines("e4m3_codes.txt"):
        v, code = line.split()[:2]
        out.append((float(v), int(code, 16)))
    return out


def fp8_block():
    chans, scale = [], None
    for line in _lines("fp8_block_hand.txt"):
        parts = line.split()
        if parts[0] == "scale":
            scale = float(parts[1])
        else:
            chans.append((int(parts[0]), float(parts[1]), int(parts[3], 16)))
    return chans, scale


def combine_case():
    d = {}
    for line in _lines("combine_hand.txt"):
        key, vals = line.split(":", 1)
        d[key.strip()] = [float(v) for v in vals.split()]
    return d


def layout_aligned_cases():
    cases, cur = [], None
    for line in _lines("layout_aligned_hand.txt"):
        if line.startswith("case"):
            T, k, E, align = map(int, line.split()[1:])
            cur = dict(T=T, k=k, E=E, align=align)
            cases.append(cur)
        else:
            key, vals = line.split(":", 1)
            cur[key.strip()] = [int(v) for v in vals.split()]
    return cases
