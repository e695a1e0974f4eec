"""Helpers for the GPU parity tests: run the oracle on the same inputs (sampled where the full
problem is large) and compare element by element."""
import numpy as np
import pytest
import torch

import oracle as O

gpu = pytest.mark.gpu


def need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def f16np(t):
    return t.detach().cpu().numpy()


def bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def check_tq_gemm(x, packed, scale, bias, y, rows=None, cols=None, label=""):
    """Compare y (GPU) with the oracle on the selected rows (tokens) and columns (outputs)."""
    K = x.shape[1]
    xs = f16np(x if rows is None else x[rows])
    p = packed.cpu().numpy()
    s = bits(scale)
    b = None if bias is None else f16np(bias)
    yt = f16np(y)
    if rows is not None:
        yt = yt[rows]
    if cols is not None:
        p, s, yt = p[cols], s[cols], yt[:, cols]
        b = None if b is None else b[cols]
    yref, bound = O.tq_gemm(xs, p, s, b, K)
    r = O.quant_check(yref, yt, bound=bound)
    assert r["ok"], (label, r)
    return r


def check_w4g_gemm(x, qweight, scales, bias, y, rows=None, cols=None, label=""):
    K = x.shape[1]
    xs = f16np(x if rows is None else x[rows])
    qw = qweight.cpu().numpy()
    s = bits(scales)
    b = None if bias is None else f16np(bias)
    yt = f16np(y)
    if rows is not None:
        yt = yt[rows]
    if cols is not None:
        qw, s, yt = qw[cols], s[cols], yt[:, cols]
        b = None if b is None else b[cols]
    yref, bound = O.w4g_gemm(xs, qw, s, b, K)
    r = O.quant_check(yref, yt, bound=bound)
    assert r["ok"], (label, r)
    return r


# Output canaries: every output buffer is allocated with guard elements on both sides, filled
# with a quiet-NaN payload no kernel writes, and checked after the call (replaces the
# sanitizer's out-of-bounds detection for the output side).
GUARD = 64               # elements (128 bytes: keeps the output 16-byte aligned)
CANARY = 0x7E5A          # quiet NaN with a payload


def guarded_empty(M, N, device="cuda"):
    """(y [M,N] fp16 view, whole buffer) with GUARD canary elements before and after y."""
    buf = torch.empty(M * N + 2 * GUARD, dtype=torch.int16, device=device)
    buf.fill_(CANARY - 0x10000 if CANARY > 0x7FFF else CANARY)
    buf = buf.view(torch.float16)
    return buf[GUARD:GUARD + M * N].view(M, N), buf


def check_canaries(buf, M, N, label=""):
    b = buf.detach().cpu().view(torch.int16).numpy().view(np.uint16)
    head, tail = b[:GUARD], b[GUARD + M * N:]
    assert (head == CANARY).all() and (tail == CANARY).all(), f"{label}: write outside y [{M},{N}]"
