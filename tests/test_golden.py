"""Fixtures under tests/golden/: what the pages print, and the oracle's own
outputs on the tiny workload as written by tests/golden/make_oracle_golden.py
(which calls only the oracle)."""
import json
import os

import numpy as np
import pytest
import torch

import oracle

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")

pytestmark = pytest.mark.usefixtures("oracle_lib")


def test_the_sdpa_pages_example_shapes_and_softmax_range():
    g = json.load(open(os.path.join(HERE, "sdpa_example_shape.json")))
    B, N, D = g["input_shape"]
    H = 8                                   # d_model = heads x head dim
    d = D // H
    gen = torch.Generator().manual_seed(3)
    q, k, v = (torch.randn(B, H, N, d, generator=gen).to(torch.bfloat16) for _ in range(3))
    rows = np.array([0, N - 1], dtype=np.int32)
    out, w = oracle.attn_exact(q, k, v, 1.0 / np.sqrt(d), rows=rows, want_weights=True)
    merged = (B, N, H * d)                  # heads concatenated back into d_model
    assert list(merged) == g["printed_output_shape"]
    assert out.shape == (B, H, len(rows), d)
    lo, hi = g["softmax_output_range"]
    assert w.min() >= lo and w.max() <= hi
    np.testing.assert_allclose(w.sum(axis=-1), 1.0, rtol=0, atol=1e-12)


def test_oracle_outputs_match_their_recorded_digests():
    import importlib.util
    spec = importlib.util.spec_from_file_location("make_oracle_golden", os.path.join(HERE, "make_oracle_golden.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    want = json.load(open(os.path.join(HERE, "oracle_tiny.json")))
    got = mod.digests()
    assert got == want
