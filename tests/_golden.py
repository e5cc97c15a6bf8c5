"""Reader for the text fixtures under tests/golden/ (``key: value`` lines, ``#`` comments)."""
import os

GOLDEN_DIR = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def load(name):
    out = {}
    with open(os.path.join(GOLDEN_DIR, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, _, val = line.partition(":")
            out[key.strip()] = val.strip()
    return out


def floats(s):
    return [float(x) for x in s.split()]


def ints(s):
    return [int(x) for x in s.split()]
