"""The decode entry point that allocates nothing (beam_attn_decode_noalloc).

It serves callers that may not allocate device memory themselves or let a
library do so -- hosts that own every byte of device memory in their own pools,
or loops where an allocation and its implied synchronisation cannot be afforded.
Its scratch is a fixed 8 MiB array inside the library, shared by all calls.

The test calls it through the C ABI twice in a row, on two different decode
problems (the second leaves stale data from the first in the shared scratch),
and compares each output with the ordinary beam_attn_decode, which gets its own
workspace, within the parity tolerance the other GPU tests use.  It also checks
that a call needing more scratch than the fixed array is rejected before any
launch.  The file sorts last so that a run stopping at the first failure has
run every other test first.
"""
import numpy as np
import pytest

import workloads as wl

pytestmark = pytest.mark.gpu

ATOL = 1e-2
RTOL = 1e-2


@pytest.fixture(scope="module")
def env():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import global_nope_gqa_b200 as beam
    beam.lib()
    return torch, beam


def _dev(torch, bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _decode_both(torch, beam, kind, ctx, slots, seed):
    params = beam.default_params()
    di = wl.decode_inputs(kind, np.array(ctx, np.int64), slots, seed, layer=f"noalloc{kind}")
    layout = beam.beam_kv_layout(kind, params, di.B, slots)
    args = [_dev(torch, x) for x in (di.q, di.k, di.v, di.gate)]
    w = [torch.from_numpy(x).cuda() for x in (di.q_norm_w, di.k_norm_w, di.gate_bias)]
    pos = torch.from_numpy(di.pos).cuda()
    outs = []
    for fn in ("beam_attn_decode", "beam_attn_decode_noalloc"):
        kc = _dev(torch, di.k_cache).view(-1)   # each call appends to its own copy
        vc = _dev(torch, di.v_cache).view(-1)
        out = torch.full((di.B, 6144), float("nan"), dtype=torch.bfloat16, device="cuda")
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        getattr(beam, fn)(kind, params, *args, *w, pos, kc, vc, layout, out, dev_status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        outs.append(out.float().cpu().numpy())
    return outs


def test_noalloc_decode_matches_decode_on_two_calls_in_a_row(env):
    torch, beam = env
    cases = [(wl.GLOBAL, [1, 700, 4097, 9000], 9000, 5),   # several splits per sequence
             (wl.LOCAL, [3, 512, 513, 2000, 70], 512, 6)]    # ring, fewer sequences
    for kind, ctx, slots, seed in cases:
        ref, got = _decode_both(torch, beam, kind, ctx, slots, seed)
        assert not np.isnan(got).any()
        bad = np.abs(got - ref) > ATOL + RTOL * np.abs(ref)
        assert not bad.any(), f"kind={kind}: {bad.sum()} elements outside tolerance"


def test_noalloc_decode_rejects_calls_beyond_the_fixed_scratch(env):
    torch, beam = env
    params = beam.default_params()
    B = 1024                       # 1024 sequences need ~38 MB of scratch: over the 8 MiB
    layout = beam.beam_kv_layout(wl.LOCAL, params, B, 512)
    assert beam.beam_decode_workspace_bytes(wl.LOCAL, params, B, layout) > 8 << 20
    kc = torch.zeros(layout.bytes_k // 2, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    q = torch.zeros((B, 6144), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((B, 1024), dtype=torch.bfloat16, device="cuda")
    w = torch.ones(128, device="cuda")
    bias = torch.zeros(48, device="cuda")
    pos = torch.zeros(B, dtype=torch.int64, device="cuda")
    out = torch.zeros_like(q)
    with pytest.raises(beam.BeamError) as e:
        beam.beam_attn_decode_noalloc(wl.LOCAL, params, q, k, k, q, w, w, bias, pos, kc, vc,
                                      layout, out)
    assert e.value.status == -8
    torch.cuda.synchronize()
    assert torch.count_nonzero(out).item() == 0 and torch.count_nonzero(kc).item() == 0
