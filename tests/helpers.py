"""Small helpers shared by the tests (fixture parsing, tolerances)."""
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def golden(name):
    """Parse a tests/golden fixture: '#' comment lines, then whitespace-separated rows."""
    rows = []
    with open(os.path.join(ROOT, "tests", "golden", name), encoding="utf-8") as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


def golden_kv(name):
    return {r[0]: r[1:] for r in golden(name)}
