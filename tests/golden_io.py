"""Readers for the text fixtures under tests/golden (no arithmetic of the method)."""
import os

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
FMT = {"fn": 0, "fnuz": 1}


def rows(name):
    """Non-comment lines of a fixture, split on '|' and stripped."""
    out = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            out.append([p.strip() for p in line.split("|")])
    return out


def floats(s):
    return [float(v) for v in s.split()]


def hexbytes(s):
    return [int(v, 16) for v in s.split()]


def matrix(s, conv):
    return [conv(r) for r in s.split(";")]
