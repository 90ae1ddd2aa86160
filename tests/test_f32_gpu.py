"""GPU parity for the QLoRA linear forward and adapter backward in the F32
compute dtype (the pages' debugging mode: rust-ai-core QLoraConfig, "Compute
Dtype"), through the C ABI, against the fp64 CPU oracle.

Reading: x, A, B, dy, bias and the outputs are fp32; the base is the fp32
dequant w' itself; every product and sum is an IEEE fp32 operation;
T = s (x A^T) and U = s (dy B) are fp32 (s is a power of two, so the scaling
is exact).  The tolerance is the worst-case bound of that arithmetic, per
element, for any summation order: an n-term fp32 dot product is within
gamma_n * sum |a_i b_i| of the exact one, gamma_n = n u / (1 - n u),
u = 2^-24 (Higham, "Accuracy and Stability of Numerical Algorithms",
section 3.1).  Errors carried in from the fp32 T and U are added through the
products that consume them:

  T:  s gamma_K |x| |A|^T                          =: eT
  y:  gamma_{K+r+1} (|x| |w'|^T + |T| |B|^T + |bias|) + eT |B|^T
  U:  s gamma_N |dy| |B|                           =: eU
  dB: gamma_M |dy|^T |T| + |dy|^T eT
  dA: gamma_M |U|^T |x| + eU^T |x|
  dx: gamma_{N+r} (|dy| |w'| + |U| |A|) + eU |A|

(|T| and |U| are taken as the exact magnitudes plus their bounds.)  That
bound is far tighter than the 16-bit tolerance, and every case also runs with
an all-zero base so the adapter path is checked on its own.
"""
import numpy as np
import pytest

from oracle import nf4_oracle as O
from qlora_linear_layers_nf4_b200 import workloads as WL

pytestmark = pytest.mark.gpu
U32 = 2.0 ** -24


def gamma(n):
    return n * U32 / (1.0 - n * U32)


def _within(name, got, want, bound):
    err = np.abs(got - want)
    excess = err - bound - 1e-30
    assert np.all(excess <= 0), (f"{name}: worst excess {np.max(excess):.3e} "
                                 f"(max err {np.max(err):.3e}, bound there {bound.flat[np.argmax(excess)]:.3e})")


def _run(case, dev, zero_w=False, bias=False, rows=None, t_from_fwd=True):
    import torch
    from qlora_linear_layers_nf4_b200 import nf4qlora as Q
    inp = WL.draw_linear(case)
    w = np.zeros_like(inp.w) if zero_w else inp.w
    ref_q = O.quantize(w, case.block_size, double=case.double_quant)
    q = Q.quantize(torch.from_numpy(w).to(dev), case.block_size, case.double_quant)
    f32 = inp.extra["f32"]
    x, A, B, dy = (torch.from_numpy(np.ascontiguousarray(f32[k])).to(dev) for k in ("x", "a", "b", "dy"))
    bias_t = bias_np = None
    if bias:
        bb = np.random.default_rng(case.seed + 99).standard_normal(case.n).astype(np.float32) * np.float32(0.1)
        bias_t, bias_np = torch.from_numpy(bb).to(dev), bb.astype(np.float64)
    ws = Q.Workspace(dev)
    y, T = Q.linear_fwd(q, x, A, B, case.alpha, bias=bias_t, workspace=ws)
    dA, dB, dx = Q.linear_bwd(q, x, A, B, case.alpha, dy, t=T if t_from_fwd else None, workspace=ws)
    torch.cuda.synchronize()
    assert ws.read_status() == 0
    assert y.dtype == torch.float32 and T.dtype == torch.float32 and dx.dtype == torch.float32

    w_hat = O.dequantize(ref_q, "f32").astype(np.float64)          # w' itself, no further rounding
    xn, an, bn, dyn = (f32[k].astype(np.float64) for k in ("x", "a", "b", "dy"))
    M, K = xn.shape
    N, r = bn.shape
    s = case.alpha / case.r
    rows = np.arange(M) if rows is None else rows
    g = lambda t: t.cpu().double().numpy()
    ax, aa, ab, ady, aw = (np.abs(v) for v in (xn, an, bn, dyn, w_hat))

    # forward
    y_ref, t_ref = O.qlora_forward(xn[rows], w_hat, an, bn, case.alpha, bias=bias_np)
    eT = s * gamma(K) * (ax @ aa.T)                                  # [M, r]
    tmag = np.abs(s * (xn @ an.T)) + eT
    _within("T", g(T)[rows], s * t_ref, eT[rows])
    b_abs = 0.0 if bias_np is None else np.abs(bias_np)[None, :]
    bound_y = gamma(K + r + 1) * (ax[rows] @ aw.T + tmag[rows] @ ab.T + b_abs) + eT[rows] @ ab.T
    _within("y", g(y)[rows], y_ref, bound_y)

    # backward
    d_a, d_b, _ = O.qlora_backward(xn, w_hat, an, bn, case.alpha, dyn)
    eU = s * gamma(N) * (ady @ ab)                                   # [M, r]
    umag = np.abs(s * (dyn @ bn)) + eU
    _within("dB", g(dB), d_b, gamma(M) * (ady.T @ tmag) + ady.T @ eT)
    _within("dA", g(dA), d_a, gamma(M) * (umag.T @ ax) + eU.T @ ax)
    _, _, d_x = O.qlora_backward(xn[rows], w_hat, an, bn, case.alpha, dyn[rows])
    bound_dx = gamma(N + r) * (ady[rows] @ aw + umag[rows] @ aa) + eU[rows] @ aa
    _within("dx", g(dx)[rows], d_x, bound_dx)


@pytest.mark.parametrize("m,n,k,rank,dq,bias", [
    (16, 256, 256, 8, False, False),       # the tiny layer
    (1, 512, 1024, 16, True, True),        # one token
    (200, 512, 512, 32, True, True),       # ragged M over two row tiles
    (300, 264, 320, 16, True, True),       # ragged M and N; K not a multiple of 128
    (512, 512, 512, 64, True, False),      # whole tiles
    (129, 136, 192, 136, False, True),     # r spanning two column tiles, one row past a tile
])
def test_f32_shapes(cuda_device, m, n, k, rank, dq, bias):
    case = WL.LinearCase(f"f32 {m}x{n}x{k} r={rank}", n=n, k=k, m=m, r=rank, alpha=2.0 * rank,
                         seed=5000 + m + n + k + rank, double_quant=dq)
    _run(case, cuda_device, bias=bias)
    _run(case, cuda_device, zero_w=True)


@pytest.mark.parametrize("bs", [128, 1024])
def test_f32_block_sizes(cuda_device, bs):
    """Blocks of 128 and 1024 over the flattened weight (they straddle rows of 320)."""
    case = WL.LinearCase(f"f32 block {bs}", n=264, k=320, m=100, r=16, alpha=32.0,
                         seed=5200 + bs, block_size=bs, double_quant=True)
    _run(case, cuda_device, bias=True)
    _run(case, cuda_device, zero_w=True)


def test_f32_recomputed_t(cuda_device):
    case = WL.LinearCase("f32 t recomputed", n=256, k=384, m=96, r=16, alpha=32.0, seed=5101,
                         double_quant=True)
    _run(case, cuda_device, t_from_fwd=False)


def test_f32_full_layer_sampled(cuda_device):
    case = WL.PREFILL
    rows = np.sort(np.random.default_rng(13).choice(case.m, 32, replace=False))
    _run(case, cuda_device, rows=rows)
