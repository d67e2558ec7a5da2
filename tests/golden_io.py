"""Readers for the hand-written fixtures under tests/golden/ (plain text, '#' comments)."""
import os

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for ln in f:
            ln = ln.strip()
            if ln and not ln.startswith("#"):
                yield ln.split()


def pairs(name):
    """[(first token, second token)] rows."""
    return [(a, b) for a, b, *_ in lines(name)]


def keyed(name):
    """{key: [tokens...]} for rows that start with a key word."""
    return {row[0]: row[1:] for row in lines(name)}
