"""Reader for tests/golden/*.txt fixtures (records: kind values... # citation)."""
import os

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def records(name):
    out = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                kind, *vals = line.split()
                out.append((kind, [float(v) for v in vals]))
    return out


def first(name, kind):
    return [v for k, v in records(name) if k == kind]
