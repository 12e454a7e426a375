"""Small text fixtures holding numbers the pages print, each with its citation
in the file's comment lines."""
import os

_HERE = os.path.dirname(os.path.abspath(__file__))


def load(name: str) -> dict:
    out = {}
    with open(os.path.join(_HERE, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, val = line.split(None, 1)
            out[key] = float(val) if any(c in val for c in ".eE") else int(val)
    return out
