"""Reader for the cited text fixtures under tests/golden/ (comment lines start with '#')."""
import os

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def rows(name):
    out = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                out.append(line.split())
    return out


def keyed(name):
    return {r[0]: r[1:] for r in rows(name)}
