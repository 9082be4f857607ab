"""Reader for the text fixtures under tests/golden/."""
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def read_sections(name):
    """Parse '[name RxC]' sections of whitespace-separated tokens."""
    sections, cur = {}, None
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            if line.startswith("["):
                cur = line.strip("[]").split()[0]
                sections[cur] = []
            else:
                sections[cur].append(line.split())
    return sections


def hex_array(rows, dtype):
    return np.array([[int(v, 16) for v in r] for r in rows], dtype=dtype)


def float_array(rows, dtype):
    return np.array([[float(v) for v in r] for r in rows], dtype=dtype)
