"""Readers for the text fixtures under tests/golden/."""
import math
import os

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield line


def _eval_e(expr):
    # expressions use only e, integers, + - * / and parentheses
    allowed = set("0123456789e+-*/(). ")
    if not set(expr) <= allowed:
        raise ValueError(expr)
    return eval(expr, {"__builtins__": {}}, {"e": math.e})


def two_frame_cases(cross_frame_special=True):
    """Cases and page tables of the two-frame example, with (default) or
    without cross-frame special retention."""
    case_tag, table_tag = ("case", "table") if cross_frame_special else ("nocross",
                                                                          "table_nocross")
    cases, tables = [], []
    for line in _lines("two_frame_example.txt"):
        head, _, vals = line.partition(":")
        tag = head.split()[0]
        kv = dict(tok.split("=") for tok in head.split()[1:])
        if tag == case_tag:
            cases.append((int(kv["S"]), int(kv["W"]), int(kv["t"]), int(kv["row"]),
                          [_eval_e(x) for x in vals.split(",")]))
        elif tag == table_tag:
            body = dict(tok.split("=") for tok in vals.split())
            tables.append((int(kv["S"]), int(kv["W"]), int(kv["t"]),
                           body["indices"].split(","), int(body["last_page_len"])))
    return cases, tables


def kv_file(name):
    out = {}
    for line in _lines(name):
        k, v = line.split("=")
        out[k.strip()] = int(v)
    return out


def visible_counts():
    out = {}
    for line in _lines("visible_counts.txt"):
        head, _, vals = line.partition(":")
        out[head.split()[0]] = (head, vals.split())
    return out
