"""Reader for the small text fixtures under tests/golden/ (key = value lines, 'case' blocks)."""
import os

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _value(v):
    parts = v.split()
    out = []
    for p in parts:
        try:
            out.append(int(p))
        except ValueError:
            try:
                out.append(float(p))
            except ValueError:
                out.append(p)
    return out[0] if len(out) == 1 else out


def load(name):
    """Return (header dict, list of case dicts) for tests/golden/<name>."""
    header, cases, cur = {}, [], None
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            if line.startswith("case "):
                cur = {"name": line[5:].strip()}
                cases.append(cur)
                continue
            key, _, val = line.partition("=")
            (cur if cur is not None else header)[key.strip()] = _value(val.strip())
    return header, cases
