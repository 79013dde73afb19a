"""Device-side failure detection: a bounded wait in the prefill attention kernel
that runs out.

The fault is injected on the host: with BEAM_FAULT_INJECT=prefill_wait_stall the
library asks the kernel's MMA issuer to begin with a wait on a barrier that
nothing ever arrives at.  Nothing faults or traps: the wait gives up after about
a second, writes BEAM_ERR_DEVICE_TIMEOUT to the caller's status word, the other
roles of the CTA see the abort flag and stop, in-flight copies are drained and
the tensor memory is freed.  The test checks the status, that no output row was
written, that the stalled call ended within a bounded time, and that the same
CUDA context then runs the same call correctly (parity with the oracle).
"""
import time

import numpy as np
import pytest

import workloads as wl
from test_gpu_parity import assert_close, env, host_bits, oracle_params, run_prefill  # noqa: F401

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("kind", [wl.GLOBAL, wl.LOCAL])
def test_prefill_wait_timeout_sets_status_and_context_survives(env, monkeypatch, kind):
    torch, beam, orc = env
    inp = wl.prefill_inputs(1, 300, 91, layer=f"timeout{kind}")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    monkeypatch.setenv("BEAM_FAULT_INJECT", "prefill_wait_stall")
    t0 = time.perf_counter()
    out, *_ = run_prefill(torch, beam, kind, inp, status=status)   # synchronises
    elapsed = time.perf_counter() - t0
    monkeypatch.delenv("BEAM_FAULT_INJECT")
    code = int(status.item())
    assert code == -4, f"status {beam.STATUS.get(code, code)}, expected BEAM_ERR_DEVICE_TIMEOUT"
    assert torch.isnan(out).all(), "a stalled kernel must not write output rows"
    assert elapsed < 30.0, f"the timed-out call took {elapsed:.1f} s"

    status.zero_()
    out, *_ = run_prefill(torch, beam, kind, inp, status=status)
    assert int(status.item()) == 0
    ref = orc.prefill(kind, oracle_params(orc, beam.default_params()), inp.q, inp.k, inp.v,
                      inp.gate, inp.q_norm_w, inp.k_norm_w, inp.gate_bias)
    assert_close(host_bits(out).reshape(ref.shape), ref, f"after timeout kind={kind}")


@pytest.mark.parametrize("kind", [wl.GLOBAL, wl.LOCAL])
def test_multi_token_decode_wait_timeout(env, monkeypatch, kind):
    """The same injected stall in the tcgen05 multi-token decode kernel (a chunk of 8
    new tokens): status -4, no output row written, then a clean call passes parity."""
    torch, beam, orc = env
    from test_gpu_chunk import oracle_chunk, run_chunk
    params = beam.default_params()
    slots = 4096 if kind == wl.GLOBAL else 512
    ci = wl.chunk_inputs(kind, 8, [3000], slots, 93, layer=f"mto{kind}")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    monkeypatch.setenv("BEAM_FAULT_INJECT", "prefill_wait_stall")
    t0 = time.perf_counter()
    out, *_ = run_chunk(torch, beam, ci, params, status)
    elapsed = time.perf_counter() - t0
    monkeypatch.delenv("BEAM_FAULT_INJECT")
    assert int(status.item()) == -4
    assert torch.isnan(out).all()
    assert elapsed < 30.0
    status.zero_()
    out, *_ = run_chunk(torch, beam, ci, params, status)
    assert int(status.item()) == 0
    ref = oracle_chunk(orc, beam, ci, params)
    assert_close(host_bits(out).reshape(ref.shape), ref, f"after timeout kind={kind}")
