"""The 52-layer decode step against the fp64 oracle, layer by layer.

The step is built and captured by the same code as the bench's 1M-context decode
measurement (bench.decode_step_layers, bench.capture_step): one call per layer in
the schedule of "Beam 1.0: Local RoPE, Global NoPE and Scalable Softmax", section
"Two attention paths in one decoder" (global layers 6, 12, ..., 48, 52; the other
43 local with a 512-slot ring), replayed as one CUDA graph.  Here the context is
4,096 visible keys instead of 1,048,576, so the oracle checks every output
element of all 52 layers; the 1M-context kernels themselves are checked in
test_gpu_parity.py and test_gpu_fp8.py.  Caches are copied to the host before
the step; the oracle reads them as they were (append first, then attend: the
new token's own row comes from its projections).
"""
import numpy as np
import pytest

import workloads as wl
from test_gpu_parity import assert_close, env, host_bits, oracle_params  # noqa: F401

pytestmark = pytest.mark.gpu

CONTEXT = 4096


@pytest.mark.parametrize("fp8", [False, True])
def test_52_layer_decode_step_matches_oracle(env, fp8):
    torch, beam, orc = env
    import bench
    layers = bench.decode_step_layers(torch, beam, CONTEXT, seed=77, fp8=fp8, tag="sched")
    assert [L.kind for L in layers] == [wl.layer_kind(i) for i in range(1, 53)]
    before = []
    for L in layers:
        slots = L.layout.slots_per_seq
        if fp8:
            before.append((L.kc.cpu().numpy().reshape(1, 8, slots, 128).copy(),
                           L.vc.cpu().numpy().reshape(1, 8, slots, 128).copy()))
        else:
            before.append((host_bits(L.kc).reshape(1, 8, slots, 128).copy(),
                           host_bits(L.vc).reshape(1, 8, slots, 128).copy()))
        L.out.fill_(float("nan"))
    graph = bench.capture_step(torch, layers)
    graph.replay()
    torch.cuda.synchronize()
    P = oracle_params(orc, beam.default_params())
    for i, (L, (k0, v0)) in enumerate(zip(layers, before), 1):
        assert int(L.status.item()) == 0, f"layer {i}"
        di = L.inputs
        if fp8:
            ref = orc.decode_fp8(L.kind, P, di.q, di.k, di.v, di.gate, di.q_norm_w, di.k_norm_w,
                                 di.gate_bias, di.pos, k0, v0, L.k_scale, L.v_scale)
        else:
            ref = orc.decode(L.kind, P, di.q, di.k, di.v, di.gate, di.q_norm_w, di.k_norm_w,
                             di.gate_bias, di.pos, k0, v0)
        assert_close(host_bits(L.out).reshape(ref.shape), ref,
                     f"layer {i} ({'global' if L.kind == wl.GLOBAL else 'local'}, fp8={fp8})")
        if not fp8:   # the new value row, bit for bit, at its slot
            t = int(di.pos[0])
            s = orc.cache_slot(L.kind, t, L.layout.slots_per_seq)
            vh = host_bits(L.vc).reshape(8, L.layout.slots_per_seq, 128)
            np.testing.assert_array_equal(vh[:, s], di.v[0].reshape(8, 128))
    del graph, layers
    torch.cuda.empty_cache()
