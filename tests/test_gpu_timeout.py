"""Bounded device-side waits ([TQ] §5.4-5.5: kernels that report failure by status, never by
hanging or trapping).

A test hook switches off the producers' activation loads and a second one shortens the wait
limit to about a millisecond.  The stage barriers that count the activation bytes then never
complete: every GEMM kernel's waits run out, the kernel skips the rest of its work and exits,
tq_device_status() reports TQ_ERR_TIMEOUT once, and the next normal call on the same context is
clean and bit-identical to the result from before the fault.  No GPU fault is involved: no TMA
copy is left in flight and every wait is bounded."""
import contextlib

import pytest
import torch

import bit_weight_only_tq_b200 as tq
import tq_inputs as I
from gpu_util import gpu, need_cuda

pytestmark = gpu

TQ_ERR_TIMEOUT = -6
LIMIT_CYCLES = 2_000_000  # ~1 ms at 1.9 GHz


@contextlib.contextmanager
def activation_loads_off():
    assert tq.lib.tq_debug_set_wait_limit(LIMIT_CYCLES) == 0
    assert tq.lib.tq_debug_skip_activation_loads(1) == 0
    try:
        yield
    finally:
        assert tq.lib.tq_debug_skip_activation_loads(0) == 0
        assert tq.lib.tq_debug_set_wait_limit(0) == 0


def _case(kind):
    if kind.startswith("w4g"):
        qw, sc = tq.w4g_quantize_pack(I.weights(384, 1024, 3, device="cuda"))
        M, path = (4, tq.PATH_DECODE) if kind == "w4g_decode" else (200, tq.PATH_PREFILL)
        x = I.activations(M, 1024, 4, device="cuda")
        return lambda y: tq.w4g_gemm(x, qw, sc, None, y=y, path=path), (M, 384)
    p, s = tq.tq_quantize_pack(I.weights(384, 1024, 1, device="cuda"))
    if kind in ("batch", "batch_tc"):
        M = 8
        x = I.activations(M, 1024, 2, device="cuda")
        ws = tq.batch_workspace()
        v = tq.BATCH_TENSOR_CORE if kind == "batch_tc" else tq.BATCH_MMA_SYNC
        return lambda y: tq.tq_gemm_batch([x], [p], [s], None, [y], workspace=ws, variant=v), (M, 384), ws
    M, path = {"decode": (1, tq.PATH_DECODE), "decode_m16": (16, tq.PATH_DECODE),
               "prefill": (256, tq.PATH_PREFILL), "prefill_splitk": (64, tq.PATH_PREFILL)}[kind]
    x = I.activations(M, 1024, 2, device="cuda")
    return lambda y: tq.tq_gemm(x, p, s, None, y=y, path=path), (M, 384)


@pytest.mark.parametrize("kind", ["decode", "decode_m16", "prefill", "prefill_splitk", "batch", "batch_tc",
                                  "w4g_decode", "w4g_prefill"])
def test_wait_runs_out_then_recovers(kind):
    need_cuda()
    case = _case(kind)
    run, (M, N) = case[0], case[1]
    ref = torch.empty(M, N, dtype=torch.float16, device="cuda")
    run(ref)
    assert tq.tq_device_status() == 0
    y = torch.zeros(M, N, dtype=torch.float16, device="cuda")
    with activation_loads_off():
        run(y)                                   # returns: the launch itself is fine
        assert tq.tq_device_status() == TQ_ERR_TIMEOUT
    assert tq.tq_device_status() == 0            # read and cleared
    if kind.startswith("batch"):                 # an aborted batch leaves its counters alone
        ws = case[2]
        n = 2 * torch.cuda.get_device_properties(0).multi_processor_count
        assert int(ws[: 4 * n].view(torch.int32).abs().sum().item()) == 0
    y2 = torch.empty(M, N, dtype=torch.float16, device="cuda")
    run(y2)
    assert tq.tq_device_status() == 0
    assert torch.equal(ref.view(torch.int16), y2.view(torch.int16))
