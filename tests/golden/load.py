"""Parser for the small text fixtures in this folder.

Format: '#' starts a comment line; every other line is 'key: values', where
values are whitespace-separated numbers and '|' separates matrix rows.
Numbers are returned as strings so a test can choose exact (Decimal) or
float parsing.
"""
import os

HERE = os.path.dirname(os.path.abspath(__file__))


def load(name):
    out = {}
    with open(os.path.join(HERE, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, _, rest = line.partition(":")
            rows = [r.split() for r in rest.split("|")]
            out[key.strip()] = rows if len(rows) > 1 else rows[0]
    return out
