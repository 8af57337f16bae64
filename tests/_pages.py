"""Reader for ``tests/golden/pages_constants.txt`` (constants printed on the LiveAnimate pages)."""
import os

_HERE = os.path.dirname(os.path.abspath(__file__))


def pages_constants() -> dict:
    out = {}
    with open(os.path.join(_HERE, "golden", "pages_constants.txt")) as f:
        for line in f:
            line = line.split("|")[0].strip()
            if not line or line.startswith("#"):
                continue
            k, v = (s.strip() for s in line.split("="))
            out[k] = v
    return out
