"""Readers for the text fixtures under tests/golden (each fixture carries its own citation)."""
import os

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _lines(name):
    with open(os.path.join(GOLDEN, name), encoding="utf-8") as f:
        for raw in f:
            line = raw.split("#", 1)[0].strip()
            if line:
                yield line


def sections(name):
    """{section: [(key, value_string), ...]} for files made of [section] headers and 'k: v' lines."""
    out, cur = {}, None
    for line in _lines(name):
        if line.startswith("[") and line.endswith("]"):
            cur = line[1:-1]
            out[cur] = []
        else:
            k, v = line.split(":", 1)
            out[cur].append((k.strip(), v.strip()))
    return out


def numbers(name="page_numbers.txt"):
    """{name: float} from 'name = value' lines."""
    out = {}
    for line in _lines(name):
        k, v = line.split("=", 1)
        out[k.strip()] = float(v.strip())
    return out
