"""GPU parity for the QLoRA linear forward and adapter backward in the F16
compute dtype (the pages list BF16, F16 and F32 as honoured compute dtypes),
through the C ABI, against the fp64 CPU oracle.

The inputs are the same seeded fp32 draws as the BF16 tests, rounded to f16;
the oracle's base is the f16 dequant (one fp32 product rounded to f16).  Same
per-tensor tolerance as BF16: max |gpu - oracle| <= 1e-2 * max |oracle|, and
every case is also run with an all-zero base so the adapter path is checked
on its own.
"""
import numpy as np
import pytest

from oracle import nf4_oracle as O
from qlora_linear_layers_nf4_b200 import workloads as WL

pytestmark = pytest.mark.gpu
TOL = 1e-2


def _close(name, got, want, tol=TOL):
    scale = np.max(np.abs(want))
    err = np.max(np.abs(got - want))
    assert err <= tol * scale, f"{name}: max err {err:.3e} vs {tol} * {scale:.3e}"


def _run(case, dev, zero_w=False, bias=False, rows=None):
    import torch
    from qlora_linear_layers_nf4_b200 import nf4qlora as Q
    inp = WL.draw_linear(case)
    w = np.zeros_like(inp.w) if zero_w else inp.w
    ref_q = O.quantize(w, 64, double=case.double_quant)
    q = Q.quantize(torch.from_numpy(w).to(dev), 64, case.double_quant)
    f16 = {k: v.astype(np.float16) for k, v in inp.extra["f32"].items()}
    x, A, B, dy = (torch.from_numpy(f16[k]).to(dev) for k in ("x", "a", "b", "dy"))
    bias_t = bias_np = None
    if bias:
        bb = (np.random.default_rng(case.seed + 99).standard_normal(case.n).astype(np.float32) * 0.1).astype(np.float16)
        bias_t, bias_np = torch.from_numpy(bb).to(dev), bb.astype(np.float64)
    ws = Q.Workspace(dev)
    y, T = Q.linear_fwd(q, x, A, B, case.alpha, bias=bias_t, workspace=ws)
    dA, dB, dx = Q.linear_bwd(q, x, A, B, case.alpha, dy, t=T, workspace=ws)
    torch.cuda.synchronize()
    assert ws.read_status() == 0
    assert y.dtype == torch.float16 and dx.dtype == torch.float16
    w_hat = O.dequantize(ref_q, "f16").astype(np.float64)
    xn, an, bn, dyn = (f16[k].astype(np.float64) for k in ("x", "a", "b", "dy"))
    rows = np.arange(xn.shape[0]) if rows is None else rows
    y_ref, t_ref = O.qlora_forward(xn[rows], w_hat, an, bn, case.alpha, bias=bias_np)
    s = case.alpha / case.r
    g = lambda t: t.float().cpu().double().numpy()
    _close("y", g(y)[rows], y_ref)
    _close("T", g(T)[rows], s * t_ref)
    d_a, d_b, _ = O.qlora_backward(xn, w_hat, an, bn, case.alpha, dyn)
    _close("dA", g(dA), d_a)
    _close("dB", g(dB), d_b)
    _, _, d_x = O.qlora_backward(xn[rows], w_hat, an, bn, case.alpha, dyn[rows])
    _close("dx", g(dx)[rows], d_x)


@pytest.mark.parametrize("m,n,k,rank,dq,bias", [
    (16, 256, 256, 8, False, False),       # decode path (mma.sync, f16 lookup table)
    (1, 512, 1024, 16, True, True),        # decode path, one token
    (17, 4096, 4096, 16, True, False),     # decode path, widest instantiation (17..32 tokens)
    (32, 1024, 2048, 16, False, True),     # decode path, 32 tokens, fp32 block scales
    (24, 512, 512, 64, True, True),        # decode path, largest decode adapter
    (200, 512, 512, 32, True, True),       # single-CTA fused kernel
    (300, 264, 320, 16, True, True),       # pair kernel, ragged M and N
    (512, 512, 512, 64, True, False),      # pair kernel, full tiles
])
def test_f16_shapes(cuda_device, m, n, k, rank, dq, bias):
    case = WL.LinearCase(f"f16 {m}x{n}x{k} r={rank}", n=n, k=k, m=m, r=rank, alpha=2.0 * rank,
                         seed=3000 + m + n + k + rank, double_quant=dq)
    _run(case, cuda_device, bias=bias)
    _run(case, cuda_device, zero_w=True)


def test_f16_full_layer_sampled(cuda_device):
    case = WL.PREFILL
    rows = np.sort(np.random.default_rng(11).choice(case.m, 48, replace=False))
    _run(case, cuda_device, rows=rows)
