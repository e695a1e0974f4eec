"""Parity at the full sizes of the benchmark configurations, in the launch configuration the
bench times (AUTO dispatch; grouped q/k/v and gate/up), checked on sampled outputs that the
oracle computes one by one, plus bit-exact packing on sampled rows."""
import numpy as np
import pytest
import torch

import bit_weight_only_tq_b200 as tq
import oracle as O
import tq_inputs as I
from gpu_util import bits, check_tq_gemm, check_w4g_gemm, gpu, need_cuda

pytestmark = gpu

LLAMA = I.LLAMA3_8B
QWEN = I.QWEN2_7B


def _sample_cols(N, k=96, seed=0):
    rng = np.random.default_rng(seed)
    return np.unique(np.concatenate([rng.choice(N, k, replace=False), [0, N - 1]]))


def _pack_layer(config, layer, shapes, dtype=torch.float32, check_rows=8):
    out = {}
    for mid, (name, (N, K)) in enumerate(shapes.items()):
        w = I.weights(N, K, I.seed_for(config, layer, mid), device="cuda", dtype=dtype)
        p, s = tq.tq_quantize_pack(w)
        rows = _sample_cols(N, check_rows, mid)
        pr, sr = O.tq_quantize_pack(w[torch.as_tensor(rows, device="cuda")].cpu().numpy())
        assert np.array_equal(p.cpu().numpy()[rows], pr), name
        assert np.array_equal(bits(s)[rows], sr), name
        out[name] = (N, K, p, s)
        del w
    return out


@pytest.mark.parametrize("M", [1, 4, 16])
def test_config1_llama_decode_full_size(M):
    need_cuda()
    L = _pack_layer(1, 31, LLAMA)
    x4 = I.activations(M, 4096, I.seed_for(1, 99, M) + 4096, device="cuda")
    x14 = I.activations(M, 14336, I.seed_for(1, 99, M) + 14336, device="cuda")
    names = list(LLAMA)
    qkv = [L[n] for n in names[0:3]]
    ys = tq.tq_gemm_grouped(x4, [v[2] for v in qkv], [v[3] for v in qkv])
    gu = [L[n] for n in names[4:6]]
    ys += tq.tq_gemm_grouped(x4, [v[2] for v in gu], [v[3] for v in gu])
    yo = tq.tq_gemm(x4, L["o_proj"][2], L["o_proj"][3])
    yd = tq.tq_gemm(x14, L["down_proj"][2], L["down_proj"][3])
    torch.cuda.synchronize()
    for (N, K, p, s), y in zip(qkv + gu, ys):
        check_tq_gemm(x4, p, s, None, y, cols=_sample_cols(N), label=f"M={M} N={N}")
    check_tq_gemm(x4, L["o_proj"][2], L["o_proj"][3], None, yo, cols=_sample_cols(4096), label="o")
    check_tq_gemm(x14, L["down_proj"][2], L["down_proj"][3], None, yd, cols=_sample_cols(4096), label="down")


@pytest.mark.parametrize("M", [512, 2048, 8192])
def test_config2_llama_prefill_full_size(M):
    need_cuda()
    L = _pack_layer(2, 0, {k: LLAMA[k] for k in ("q_proj", "k_proj", "gate_proj", "down_proj")})
    rng = np.random.default_rng(M)
    for name, (N, K, p, s) in L.items():
        x = I.activations(M, K, I.seed_for(2, 0, K), device="cuda", outlier_row_frac=0.01)
        b = I.bias(N, I.seed_for(2, 1, N), device="cuda")
        y = tq.tq_gemm(x, p, s, b)
        torch.cuda.synchronize()
        # sampled token rows (including outlier rows) x sampled output columns
        norms = x.float().abs().amax(dim=1)
        outl = torch.nonzero(norms > 30).flatten().cpu().numpy()[:4]
        rows = np.unique(np.concatenate([rng.choice(M, 12, replace=False), outl, [M - 1]]))
        check_tq_gemm(x, p, s, b, y, rows=rows, cols=_sample_cols(N, 64), label=f"{name} M={M}")


@pytest.mark.parametrize("M", [1, 16, 256, 4096])
def test_config3_w4g_full_size(M):
    need_cuda()
    for mid, name in ((0, "q_proj"), (4, "gate_proj"), (6, "down_proj")):
        N, K = LLAMA[name]
        w = I.weights(N, K, I.seed_for(3, 0, mid), device="cuda", outlier_frac=0.001)
        qw, sc = tq.w4g_quantize_pack(w)
        rows = _sample_cols(N, 6, mid)
        qr, sr = O.w4g_quantize_pack(w[torch.as_tensor(rows, device="cuda")].cpu().numpy())
        assert np.array_equal(qw.cpu().numpy()[rows], qr) and np.array_equal(bits(sc)[rows], sr)
        del w
        x = I.activations(M, K, I.seed_for(3, 2, K) + M, device="cuda")
        y = tq.w4g_gemm(x, qw, sc)
        torch.cuda.synchronize()
        trows = None if M <= 16 else np.random.default_rng(M).choice(M, 12, replace=False)
        check_w4g_gemm(x, qw, sc, None, y, rows=trows, cols=_sample_cols(N, 64), label=f"w4g {name} M={M}")


def test_config4_qwen_fp16_pack_and_m_sweep():
    need_cuda()
    L = _pack_layer(4, 0, QWEN, dtype=torch.float16, check_rows=16)
    for M in (1, 2, 8, 32, 128, 512, 2048, 8192):
        for name, (N, K, p, s) in L.items():
            x = I.activations(M, K, I.seed_for(4, 1, M) + K, device="cuda")
            y = tq.tq_gemm(x, p, s)
            torch.cuda.synchronize()
            trows = None if M <= 16 else np.random.default_rng(M + K).choice(M, 8, replace=False)
            check_tq_gemm(x, p, s, None, y, rows=trows, cols=_sample_cols(N, 32), label=f"qwen {name} M={M}")
