"""Readers for the cited text fixtures under tests/golden/ (values as the pages print them)."""
import os

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def read(name):
    """Return (scalars: dict key -> list of str, rows: list of lists of str)."""
    scalars, rows = {}, []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = line.split()
            if parts[0] == "row":
                rows.append(parts[1:])
            else:
                scalars.setdefault(parts[0], []).append(parts[1:])
    return scalars, rows


def scalar(scalars, key):
    return float(scalars[key][0][0])
