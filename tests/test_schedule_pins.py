"""The 52-layer attention schedule of the decode step, pinned to the pages.

Source: "Beam 1.0: Local RoPE, Global NoPE and Scalable Softmax" (flozi.net),
section "Two attention paths in one decoder" (the list of global layers) and
section "KV memory: nine growing caches, not 52" (nine growing caches).  The
input module's schedule drives every 52-layer measurement and the 52-layer
parity test; a slip in it (a layer off by one, a missing last layer) would
change every 1M-context number without failing any kernel test.
"""
import os

import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "layer_schedule.txt")


def _golden():
    out = {}
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                key, *vals = line.split()
                out[key] = [int(v) for v in vals]
    return out


def test_global_layers_match_the_printed_list():
    g = _golden()
    assert wl.N_LAYERS == g["n_layers"][0]
    assert wl.WINDOW == g["window"][0]
    assert tuple(wl.GLOBAL_LAYERS) == tuple(g["global"])
    kinds = [wl.layer_kind(i) for i in range(1, wl.N_LAYERS + 1)]
    assert [i for i, k in enumerate(kinds, 1) if k == wl.GLOBAL] == g["global"]
    assert kinds.count(wl.GLOBAL) == g["n_global"][0]
    assert kinds.count(wl.LOCAL) == g["n_local"][0]


def test_global_layers_are_every_sixth_plus_the_last():
    """The Arabic page's description of the same set, derived independently."""
    derived = sorted({i for i in range(1, 53) if i % 6 == 0} | {52})
    assert derived == list(wl.GLOBAL_LAYERS)
    assert wl.layer_kind(0 + 1) == wl.LOCAL and wl.layer_kind(52) == wl.GLOBAL
    assert wl.layer_kind(51) == wl.LOCAL and wl.layer_kind(53) == wl.LOCAL


def test_decode_workload_runs_the_schedule():
    """The 1M-context decode workload runs one call per layer in this order."""
    w = wl.workload("decode_1m")
    assert len(w.layers) == 52
    assert [i for i, k in enumerate(w.layers, 1) if k == wl.GLOBAL] == _golden()["global"]
    # nine growing caches of 4 KiB per token in bf16: 36 KiB per token
    # (section "KV memory: nine growing caches, not 52")
    per_token = sum(2 * wl.N_KV_HEADS * wl.HEAD_DIM * 2 for k in w.layers if k == wl.GLOBAL)
    assert per_token == 36 * 1024
