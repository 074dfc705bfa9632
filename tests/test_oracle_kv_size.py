"""Pins the KV-size closed form to the figures the pages print."""
import os

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    with open(os.path.join(GOLD, name)) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                yield line.split()


def test_exact_bytes_per_token():
    for layers, tokens, kvh, hd, nbytes, expected in _rows("kv_size.txt"):
        assert oracle.kv_bytes(int(layers), int(tokens), int(kvh), int(hd), int(nbytes)) == int(
            expected)


def test_rounded_request_size():
    for layers, tokens, kvh, hd, nbytes, printed_gb, digits in _rows("kv_size_approx.txt"):
        got = oracle.kv_bytes(int(layers), int(tokens), int(kvh), int(hd), int(nbytes)) / 1e9
        assert float(f"{got:.{int(digits)}g}") == float(printed_gb)


def test_mha_over_gqa_ratio_matches_printed_pair():
    for kva, kvb, pa, pb in _rows("kv_ratio.txt"):
        a = oracle.kv_bytes(80, 32768, int(kva), 128, 2)
        b = oracle.kv_bytes(80, 32768, int(kvb), 128, 2)
        assert b / a == float(pb) / float(pa)


def test_linearity_in_every_factor():
    base = oracle.kv_bytes(3, 5, 7, 64, 2)
    assert oracle.kv_bytes(6, 5, 7, 64, 2) == 2 * base
    assert oracle.kv_bytes(3, 10, 7, 64, 2) == 2 * base
    assert oracle.kv_bytes(3, 5, 14, 64, 2) == 2 * base
    assert oracle.kv_bytes(3, 5, 7, 128, 2) == 2 * base
    assert oracle.kv_bytes(3, 5, 7, 64, 4) == 2 * base
    assert oracle.kv_bytes(1, 1, 1, 1, 1) == 2  # the key and the value
    assert oracle.kv_bytes(3, 0, 7, 64, 2) == 0
