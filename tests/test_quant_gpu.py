"""GPU parity: NF4 quantize / double quant / dequantize, bit for bit against the
CPU oracle on the same seeded inputs, through the C ABI."""
import numpy as np
import pytest

from oracle import nf4_oracle as O
from qlora_linear_layers_nf4_b200 import workloads as WL

pytestmark = pytest.mark.gpu


def _q():
    from qlora_linear_layers_nf4_b200 import nf4qlora as Q
    return Q


def _to_dev(a, dev):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev)


def _check_quant(w, bs, dq, dev):
    Q = _q()
    import torch
    ref = O.quantize(w, bs, double=dq)
    q = Q.quantize(_to_dev(w, dev), block_size=bs, double_quant=dq, keep_absmax=True,
                   check_status=True)
    torch.cuda.synchronize()
    codes = q.codes.cpu().numpy()[: ref["codes"].size]
    assert np.array_equal(codes, ref["codes"]), "packed codes differ"
    assert np.array_equal(q.absmax.cpu().numpy()[: ref["absmax"].size].view(np.uint32),
                          ref["absmax"].view(np.uint32))
    if dq:
        assert np.array_equal(q.absmax_q.cpu().numpy()[: ref["absmax_q"].size], ref["absmax_q"])
        assert q.absmax_scale.cpu().numpy()[0].view(np.uint32) == np.float32(ref["absmax_scale"]).view(np.uint32)
    return q, ref


def _check_dequant(q, ref, dev):
    Q = _q()
    for kind in ("f32", "bf16", "f16"):
        got = Q.dequantize(q, kind).cpu()
        want = O.dequantize(ref, kind)
        if kind == "f32":
            assert np.array_equal(got.numpy().view(np.uint32), want.reshape(got.shape).view(np.uint32))
        elif kind == "bf16":
            import torch
            g = got.view(torch.int16).numpy().view(np.uint16)
            assert np.array_equal(g, want.reshape(g.shape))
        else:
            assert np.array_equal(got.numpy().view(np.uint16), want.reshape(got.shape).view(np.uint16))


def test_tiny_layer_weight(cuda_device):
    inp = WL.draw_linear(WL.TINY)
    q, ref = _check_quant(inp.w, 64, False, cuda_device)
    _check_dequant(q, ref, cuda_device)


@pytest.mark.parametrize("dq", [False, True])
def test_full_4096_square(cuda_device, dq):
    w = WL.draw_weight(WL.QUANT_SHAPE, WL.QUANT_SEED)
    q, ref = _check_quant(w, 64, dq, cuda_device)
    _check_dequant(q, ref, cuda_device)


@pytest.mark.parametrize("bs", [8, 16, 32, 128, 256, 2, 6, 24, 40, 512])
def test_block_sizes_and_ragged_grid(cuda_device, bs):
    # 7 rows x (bs * 37) columns: the element count is not a multiple of the
    # launch width, and non-power-of-two sizes take the per-block path.
    w = WL.draw_weight((7, bs * 37), seed=100 + bs)
    q, ref = _check_quant(w, bs, True, cuda_device)
    if bs % 8 == 0:
        _check_dequant(q, ref, cuda_device)


def test_edge_values(cuda_device):
    lv = O.nf4_levels()
    rng = np.random.default_rng(7)
    blocks = []
    # exact midpoints and neighbours, scaled by powers of two (absmax = 2^e)
    from fractions import Fraction
    mids = []
    for i in range(15):
        m = np.float32(float((Fraction(float(lv[i])) + Fraction(float(lv[i + 1]))) / 2))
        mids += [m, np.nextafter(m, np.float32(2)), np.nextafter(m, np.float32(-2))]
    mids = np.array(mids, dtype=np.float32)
    for e in (-10, -3, 0, 5):
        blk = np.resize(mids, 63).astype(np.float32) * np.float32(2.0 ** e)
        blocks.append(np.concatenate([blk, [np.float32(2.0 ** e)]]))
    blocks.append(np.zeros(64, np.float32))                          # absmax 0
    z = np.zeros(64, np.float32)
    z[5] = -0.0
    z[9] = np.float32(-3e-3)
    blocks.append(z)                                                 # negative absmax element
    blocks.append(np.full(64, np.float32(1e-38)))                    # tiny values
    d = np.zeros(64, np.float32)
    d[0] = np.float32(1e-42)                                         # denormal absmax
    d[1] = np.float32(-7e-43)
    blocks.append(d)
    blocks.append(rng.permutation(np.resize(lv, 64)).astype(np.float32) * np.float32(3.0))
    # block scales outside the fast-reciprocal range (above 2^120, below 2^-120)
    big = np.resize(mids, 63).astype(np.float32) * np.float32(2.0 ** 124)
    blocks.append(np.concatenate([big, [np.float32(2.0 ** 124)]]))
    small = np.resize(mids, 63).astype(np.float32) * np.float32(2.0 ** -122)
    blocks.append(np.concatenate([small, [np.float32(2.0 ** -122)]]))
    w = np.stack(blocks)
    for dq in (False, True):
        q, ref = _check_quant(w, 64, dq, cuda_device)
        _check_dequant(q, ref, cuda_device)


def test_small_block_scales_near_thresholds(cuda_device):
    # Block scales a with arbitrary significands in the lowest binades, both
    # sides of the 2^-98 edge where the kernel's division-free quotient stops
    # being exact, and elements RN(t a) for every decision threshold t and its
    # neighbours: quotients that sit on or next to a threshold, where one ulp
    # decides the code.
    rng = np.random.default_rng(31)
    _, th = _q().codebook()
    th = np.array(th, dtype=np.float32)
    ts = np.concatenate([th, np.nextafter(th, np.float32(2)), np.nextafter(th, np.float32(-2))])
    blocks = []
    for e in list(range(-125, -90)) + [-60, -20, 0, 40, 100, 118, 119]:
        for _ in range(40):
            a = np.float32((1.0 + rng.random()) * 2.0 ** e)
            vals = (np.resize(rng.permutation(ts), 63).astype(np.float64) * float(a)).astype(np.float32)
            blocks.append(np.concatenate([vals, [a]]).astype(np.float32))
    w = np.stack(blocks)
    for dq in (False, True):
        q, ref = _check_quant(w, 64, dq, cuda_device)
        _check_dequant(q, ref, cuda_device)


def test_absmax_element_exact(cuda_device):
    # values a for which multiplying by a reciprocal would not give exactly 1
    rng = np.random.default_rng(5)
    a = (rng.random(200000, dtype=np.float32) * np.float32(0.1) + np.float32(1e-3)).astype(np.float32)
    bad = a[(a * (np.float32(1.0) / a)).astype(np.float32) != np.float32(1.0)][:256]
    blocks = rng.standard_normal((bad.size, 64)).astype(np.float32) * np.float32(1e-4)
    blocks[:, 17] = bad
    blocks[::2, 17] *= -1
    q, ref = _check_quant(blocks, 64, False, cuda_device)
    _check_dequant(q, ref, cuda_device)


def test_all_zero_and_single_block(cuda_device):
    for shape in [(32, 32), (1, 64), (2, 2)]:
        w = np.zeros(shape, np.float32)
        bs = 64 if w.size % 64 == 0 else 4
        q, ref = _check_quant(w, bs, True, cuda_device)


def test_nonfinite_is_flagged(cuda_device):
    Q = _q()
    import torch
    w = WL.draw_weight((16, 64), seed=3)
    w[3, 5] = np.nan
    ws = Q.Workspace(cuda_device)
    Q.quantize(_to_dev(w, cuda_device), 64, False, workspace=ws)
    assert ws.read_status() == 7
    assert ws.read_status() == 0            # read clears it
    w[3, 5] = np.inf
    Q.quantize(_to_dev(w, cuda_device), 64, True, workspace=ws)
    assert ws.read_status() == 7


def test_empty_input(cuda_device):
    Q = _q()
    import torch
    q = Q.quantize(torch.zeros((0, 64), dtype=torch.float32, device=cuda_device), 64, True)
    torch.cuda.synchronize()
    assert q.absmax_scale.item() == 0.0


@pytest.mark.parametrize("dq", [False, True])
def test_chained_calls_without_sync(cuda_device, dq):
    """Quantize and dequantize back to back on one stream, each call reading the
    previous call's output and the quantize calls sharing one workspace, with no
    synchronisation in between (the kernels are launched as programmatic
    dependents of one another): every round is bit-exact against the oracle's
    own chain of the same rounds."""
    import torch
    Q = _q()
    w = WL.draw_weight((1024, 1024), seed=31)
    rounds = 4
    qs, outs = [], []
    cur = _to_dev(w, cuda_device)
    for _ in range(rounds):
        q = Q.quantize(cur, block_size=64, double_quant=dq, keep_absmax=True)
        cur = Q.dequantize(q, "f32")
        qs.append(q)
        outs.append(cur)
    torch.cuda.synchronize()
    ref_w = w
    for k in range(rounds):
        ref = O.quantize(ref_w, 64, double=dq)
        q = qs[k]
        assert np.array_equal(q.codes.cpu().numpy()[: ref["codes"].size], ref["codes"]), f"round {k}: codes"
        assert np.array_equal(q.absmax.cpu().numpy()[: ref["absmax"].size].view(np.uint32),
                              ref["absmax"].view(np.uint32)), f"round {k}: absmax"
        if dq:
            assert np.array_equal(q.absmax_q.cpu().numpy()[: ref["absmax_q"].size], ref["absmax_q"])
            assert q.absmax_scale.cpu().numpy()[0].view(np.uint32) == np.float32(ref["absmax_scale"]).view(np.uint32)
        ref_w = O.dequantize(ref, "f32").reshape(w.shape)
        assert np.array_equal(outs[k].cpu().numpy().view(np.uint32), ref_w.view(np.uint32)), f"round {k}: dequant"
