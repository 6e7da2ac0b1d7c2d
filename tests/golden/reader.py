"""Reads the small `key: values` text fixtures of this folder (comments start with #)."""
import os

HERE = os.path.dirname(os.path.abspath(__file__))


def load(name):
    out = {}
    with open(os.path.join(HERE, name), encoding="utf-8") as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, _, val = line.partition(":")
            out[key.strip()] = val.strip()
    return out


def floats(s):
    return [float(v) for v in s.split()]


def ints(s):
    return [int(v) for v in s.split()]
