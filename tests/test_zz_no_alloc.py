"""The decode entry point that allocates nothing (beam_attn_decode_noalloc).

It serves callers that may not allocate device memory themselves or let a
library do so -- hosts that own every byte of device memory in their own pools,
or loops where an allocation and its implied synchronisation cannot be afforded.
Its scratch is a fixed 8 MiB array inside the library, shared by all calls.

The tests call it through the C ABI twice in a row, on two different decode
problems (the second meets whatever the first left in the shared scratch), and
compare each output element by element with the fp64 oracle and with the
ordinary beam_attn_decode (which gets its own workspace), at the parity bar of
the other GPU tests.  A local layer keeps nothing in the scratch, so a local
call of any batch is accepted (checked at 400 sequences against the oracle);
a global call whose split-K partials would not fit the fixed array is rejected
before any launch, with nothing written.  The file sorts last so that a run
stopping at the first failure has run every other test first.
"""
import numpy as np
import pytest

import workloads as wl
from test_gpu_parity import assert_close, dev, env, host_bits, oracle_params  # noqa: F401

pytestmark = pytest.mark.gpu

ATOL = 1e-2
RTOL = 1e-2


def _decode_both(torch, beam, di, kc0, vc0):
    """The same decode through beam_attn_decode and beam_attn_decode_noalloc, each on
    its own copy of the caches (the call appends the new row); outputs as bf16 bits."""
    params = beam.default_params()
    layout = beam.beam_kv_layout(di.kind, params, di.B, di.slots)
    args = [dev(torch, x) for x in (di.q, di.k, di.v, di.gate)]
    w = [torch.from_numpy(x).cuda() for x in (di.q_norm_w, di.k_norm_w, di.gate_bias)]
    pos = torch.from_numpy(di.pos).cuda()
    outs = []
    for fn in ("beam_attn_decode", "beam_attn_decode_noalloc"):
        kc, vc = kc0.clone(), vc0.clone()
        out = torch.full((di.B, 6144), float("nan"), dtype=torch.bfloat16, device="cuda")
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        getattr(beam, fn)(di.kind, params, *args, *w, pos, kc, vc, layout, out, dev_status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0, fn
        outs.append(host_bits(out))
        del kc, vc
    return outs


def _check_against_oracle_and_decode(orc, beam, di, k0, v0, outs, what):
    ref = orc.decode(di.kind, oracle_params(orc, beam.default_params()), di.q, di.k, di.v,
                     di.gate, di.q_norm_w, di.k_norm_w, di.gate_bias, di.pos, k0, v0)
    plain, noalloc = outs
    assert_close(noalloc.reshape(ref.shape), ref, f"{what}: no-alloc decode vs oracle")
    assert_close(plain.reshape(ref.shape), ref, f"{what}: decode vs oracle")
    a = wl.bf16_bits_to_f32(noalloc).astype(np.float64)
    b = wl.bf16_bits_to_f32(plain).astype(np.float64)
    assert not np.isnan(a).any()
    assert not (np.abs(a - b) > ATOL + RTOL * np.abs(b)).any(), f"{what}: no-alloc vs decode"


def test_noalloc_decode_matches_oracle_on_two_calls_in_a_row(env):
    torch, beam, orc = env
    cases = [(wl.GLOBAL, [1, 700, 4097, 9000], 9000, 5),   # several splits per sequence
             (wl.LOCAL, [3, 512, 513, 2000, 70], 512, 6)]    # ring, fewer sequences
    for kind, ctx, slots, seed in cases:
        di = wl.decode_inputs(kind, np.array(ctx, np.int64), slots, seed, layer=f"noalloc{kind}")
        kc0 = dev(torch, di.k_cache).view(-1)
        vc0 = dev(torch, di.v_cache).view(-1)
        outs = _decode_both(torch, beam, di, kc0, vc0)
        _check_against_oracle_and_decode(orc, beam, di, di.k_cache, di.v_cache, outs,
                                         f"kind={kind}")


def test_noalloc_local_decode_takes_any_batch(env):
    """400 sequences of a local layer: more than a global layer's partials of that batch
    would need in the fixed scratch, yet the ring decode keeps none there."""
    torch, beam, orc = env
    params = beam.default_params()
    B = 400
    ctx = 1 + np.random.default_rng(9).integers(0, 3000, B)   # some rings full, some not
    di = wl.decode_inputs(wl.LOCAL, ctx, 512, 12, layer="noallocB", with_cache=False)
    layout = beam.beam_kv_layout(wl.LOCAL, params, B, 512)
    kc0 = torch.empty(layout.bytes_k // 2, dtype=torch.bfloat16, device="cuda")
    vc0 = torch.empty_like(kc0)
    wl.device_normal_bf16_(kc0, 12, "noallocB/kc")
    wl.device_normal_bf16_(vc0, 12, "noallocB/vc")
    shape = (B, 8, 512, 128)
    k0, v0 = host_bits(kc0).reshape(shape), host_bits(vc0).reshape(shape)
    outs = _decode_both(torch, beam, di, kc0, vc0)
    _check_against_oracle_and_decode(orc, beam, di, k0, v0, outs, "local B=400")


def test_noalloc_decode_rejects_calls_beyond_the_fixed_scratch(env):
    """640 sequences of a global layer need ~16 MB of split-K partials: more than the
    fixed 8 MiB, so the call returns BEAM_ERR_SCRATCH_LIMIT and writes nothing."""
    torch, beam, _ = env
    params = beam.default_params()
    B = 640
    layout = beam.beam_kv_layout(wl.GLOBAL, params, B, 512)
    assert beam.beam_decode_workspace_bytes(wl.GLOBAL, params, B, layout) > 8 << 20
    kc = torch.zeros(layout.bytes_k // 2, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    q = torch.zeros((B, 6144), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((B, 1024), dtype=torch.bfloat16, device="cuda")
    w = torch.ones(128, device="cuda")
    bias = torch.zeros(48, device="cuda")
    pos = torch.full((B,), 100, dtype=torch.int64, device="cuda")
    out = torch.zeros_like(q)
    with pytest.raises(beam.BeamError) as e:
        beam.beam_attn_decode_noalloc(wl.GLOBAL, params, q, k, k, q, w, w, bias, pos, kc, vc,
                                      layout, out)
    assert e.value.status == -8
    torch.cuda.synchronize()
    assert torch.count_nonzero(out).item() == 0 and torch.count_nonzero(kc).item() == 0
