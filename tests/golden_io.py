"""Reader for the ``key = value`` golden fixtures under ``tests/golden``."""

import os

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def read_golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, value = (p.strip() for p in line.split("=", 1))
            if "," in value:
                out[key] = [float(x) if "." in x else int(x) for x in value.split(",")]
            else:
                out[key] = float(value) if "." in value else int(value)
    return out
