"""Regression pins: the oracle still produces the stored tiny-layer fixtures."""
import json
import os

import numpy as np
import pytest

from oracle import hstu_layer

import importlib.util

HERE = os.path.join(os.path.dirname(__file__), "golden")
_spec = importlib.util.spec_from_file_location("make_golden", os.path.join(HERE, "make_golden.py"))
make_golden = importlib.util.module_from_spec(_spec)
_spec.loader.exec_module(make_golden)


@pytest.mark.parametrize("mask", ["causal", "mfalcon"])
def test_oracle_reproduces_fixture(mask):
    X, offs, ts, nc, p, cfg = make_golden.tiny_inputs(mask)
    out = hstu_layer(X, offs, ts, nc, p, cfg)
    with open(os.path.join(HERE, f"tiny_layer_{mask}.json")) as f:
        g = json.load(f)
    assert np.max(np.abs(out["O"] - np.array(g["O"]))) < 1e-14
    assert np.max(np.abs(out["Y"] - np.array(g["Y"]))) < 1e-13
