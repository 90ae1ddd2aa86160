"""GPU parity for the dense merge W' + (alpha/r) B A, through the C ABI,
against the CPU oracle on the same seeded inputs.

Bound per element (both outputs are one rounding of an fp32 value):
  fp32: |gpu - exact| <= 2^-23 |exact| + (r + 2) 2^-24 s (|B| |A|)
        (the fp32 rounding of the sum plus the fp32 accumulation of r exact
        bf16 x bf16 products);
  bf16: |gpu - exact| <= ulp_bf16(exact) + the fp32 bound above;
  f16:  |gpu - exact| <= ulp_f16(exact) + the fp32 bound above (normal range).
With B = 0 the merge is the plain dequant and must match it bit for bit.
"""
import numpy as np
import pytest

from oracle import nf4_oracle as O
from qlora_linear_layers_nf4_b200 import workloads as WL

pytestmark = pytest.mark.gpu


def _Q():
    from qlora_linear_layers_nf4_b200 import nf4qlora as Q
    return Q


def _bf(dev, bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)


def _run(case, dev, zero_w=False, zero_b=False, rows=None):
    import torch
    Q = _Q()
    inp = WL.draw_linear(case)
    w = np.zeros_like(inp.w) if zero_w else inp.w
    b = np.zeros_like(inp.b) if zero_b else inp.b
    ref_q = O.quantize(w, case.block_size, double=case.double_quant)
    q = Q.quantize(torch.from_numpy(w).to(dev), case.block_size, case.double_quant)
    A, B = _bf(dev, inp.a), _bf(dev, b)
    ws = Q.Workspace(dev)
    out_bf = Q.merge(q, A, B, case.alpha, "bf16", workspace=ws)
    out_f32 = Q.merge(q, A, B, case.alpha, "f32", workspace=ws)
    out_h = Q.merge(q, A, B, case.alpha, "f16", workspace=ws)
    torch.cuda.synchronize()
    assert ws.read_status() == 0
    _run.last_f16 = out_h
    return inp, ref_q, b, out_bf, out_f32


def _check(case, inp, ref_q, b_bits, out_bf, out_f32, rows=None):
    f = WL.bf16_bits_to_f32
    a, b = f(inp.a).astype(np.float64), f(b_bits).astype(np.float64)
    sel = slice(None) if rows is None else rows
    qsel = ref_q if rows is None else _rows_of(ref_q, rows)
    exact = O.merge(qsel, a, b[sel], case.alpha, "f64")
    s = case.alpha / case.r
    bound32 = 2.0 ** -23 * np.abs(exact) + (case.r + 2) * 2.0 ** -24 * s * (np.abs(b[sel]) @ np.abs(a))
    g32 = out_f32.cpu().numpy()[sel].astype(np.float64)
    assert np.all(np.abs(g32 - exact) <= bound32), f"f32: worst excess {np.max(np.abs(g32 - exact) - bound32):.3e}"
    gbf = out_bf.float().cpu().numpy()[sel].astype(np.float64)
    ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(exact), 1e-38))) - 7)
    assert np.all(np.abs(gbf - exact) <= ulp + bound32), "bf16 outside one ulp"
    # most elements are the exact bf16 rounding of the oracle's fp32 value
    want_bits = O.merge(qsel, a, b[sel], case.alpha, "bf16")
    got_bits = out_bf.cpu().view(__import__("torch").int16).numpy()[sel].view(np.uint16)
    assert np.mean(got_bits == want_bits) > 0.999
    # the f16 output of the same call: one f16 ulp plus the fp32 bound, and
    # almost always the f16 rounding of the oracle's fp32 value
    gh = _run.last_f16.cpu().numpy()[sel]
    assert np.all(np.isfinite(gh))
    ulp_h = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(exact), 2.0 ** -14))) - 10)
    assert np.all(np.abs(gh.astype(np.float64) - exact) <= ulp_h + bound32), "f16 outside one ulp"
    want_h = O.merge(qsel, a, b[sel], case.alpha, "f16")
    assert np.mean(gh.view(np.uint16) == want_h.view(np.uint16)) > 0.999


def _rows_of(q, rows):
    """The quantized rows `rows` of q as a quantized tensor of their own."""
    n, k = q["shape"]
    bs = q["block_size"]
    kb = k // bs
    codes = q["codes"].reshape(n, k // 2)[rows].reshape(-1)
    out = dict(q)
    out["codes"] = codes
    out["shape"] = (len(rows), k)
    if q.get("absmax") is not None:
        out["absmax"] = q["absmax"].reshape(n, kb)[rows].reshape(-1)
    if q.get("absmax_q") is not None:
        out["absmax_q"] = q["absmax_q"].reshape(n, kb)[rows].reshape(-1)
    return out


def test_tiny(cuda_device):
    case = WL.TINY
    _check(case, *_run(case, cuda_device))


@pytest.mark.parametrize("n,k,rank,dq", [
    (264, 320, 16, True),      # N, K not multiples of the 128 x 256 tile
    (512, 512, 64, True),
    (1032, 192, 24, False),    # r not a multiple of 16
    (256, 4096, 8, True),      # smallest rank, long rows
    (384, 1024, 136, True),    # r spanning three 64-wide chunks
    (128, 512, 256, False),    # the largest rank
])
def test_ragged_shapes(cuda_device, n, k, rank, dq):
    case = WL.LinearCase(f"merge {n}x{k} r={rank}", n=n, k=k, m=1, r=rank, alpha=2.0 * rank,
                         seed=2000 + n + k + rank, double_quant=dq)
    _check(case, *_run(case, cuda_device))


def test_b_zero_is_the_dequant_bit_for_bit(cuda_device):
    import torch
    case = WL.LinearCase("merge B=0", n=512, k=1024, m=1, r=64, alpha=128.0, seed=31)
    inp, ref_q, b, out_bf, out_f32 = _run(case, cuda_device, zero_b=True)
    assert np.array_equal(out_f32.cpu().numpy().view(np.uint32),
                          O.dequantize(ref_q, "f32").view(np.uint32))
    assert np.array_equal(out_bf.cpu().view(torch.int16).numpy().view(np.uint16),
                          O.dequantize(ref_q, "bf16"))
    assert np.array_equal(_run.last_f16.cpu().numpy().view(np.uint16),
                          O.dequantize(ref_q, "f16").view(np.uint16))


@pytest.mark.parametrize("bs,k", [(128, 512), (256, 320), (1024, 4096)])
def test_block_sizes(cuda_device, bs, k):
    """Blocks of 128 to 1024 elements (straddling rows when K is not a multiple)."""
    case = WL.LinearCase(f"merge block {bs}", n=264, k=k, m=1, r=32, alpha=64.0, seed=2100 + bs,
                         block_size=bs)
    _check(case, *_run(case, cuda_device))


def test_zero_base_leaves_the_update(cuda_device):
    case = WL.LinearCase("merge W=0", n=256, k=512, m=1, r=32, alpha=64.0, seed=32)
    _check(case, *_run(case, cuda_device, zero_w=True))


def test_full_layer_sampled_rows(cuda_device):
    case = WL.PREFILL
    inp, ref_q, b, out_bf, out_f32 = _run(case, cuda_device)
    rows = np.sort(np.random.default_rng(5).choice(case.n, 96, replace=False))
    rows = np.concatenate([rows, [0, case.n - 1]])
    _check(case, inp, ref_q, b, out_bf, out_f32, rows=rows)
