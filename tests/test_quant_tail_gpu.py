"""GPU parity for tensors whose size is not a multiple of the block size, and
for block sizes the vectorized kernels do not take: quantize (codes, scales,
double quant) and dequantize (fp32, bf16, f16), bit for bit against the CPU
oracle.

The pages' quantize_nf4 (qlora-rs README, "Honest capability matrix": NF4
pack/unpack + block absmax scales) takes a tensor of any size.  The reading
followed on both sides: the last block holds the elements that remain, its
absmax is the max over those alone, and an odd element count leaves the last
byte's low nibble at code 7 (the exact-zero level).
"""
import numpy as np
import pytest

from oracle import nf4_oracle as O
from qlora_linear_layers_nf4_b200 import workloads as WL

pytestmark = pytest.mark.gpu


def _as_input(w32, kind):
    """(fp32 values the oracle quantizes, torch tensor the GPU quantizes)."""
    import torch
    if kind == "f32":
        return w32, torch.from_numpy(w32)
    if kind == "bf16":
        bits = WL.to_bf16_bits(w32)
        t = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)
        return WL.bf16_bits_to_f32(bits).reshape(w32.shape), t.reshape(w32.shape)
    h = w32.astype(np.float16)
    return h.astype(np.float32), torch.from_numpy(h)


def _check(w32, bs, dq, dev, kind="f32"):
    import torch
    from qlora_linear_layers_nf4_b200 import nf4qlora as Q
    vals, t = _as_input(w32, kind)
    ref = O.quantize(vals, bs, double=dq)
    q = Q.quantize(t.to(dev), bs, dq, keep_absmax=True, check_status=True)
    torch.cuda.synchronize()
    numel = w32.size
    nblocks = -(-numel // bs)
    assert ref["codes"].size == (numel + 1) // 2 and ref["absmax"].size == nblocks
    assert q.codes.numel() == (numel + 1) // 2
    assert np.array_equal(q.codes.cpu().numpy(), ref["codes"]), "codes differ"
    assert np.array_equal(q.absmax.cpu().numpy().view(np.uint32), ref["absmax"].view(np.uint32))
    if dq:
        assert np.array_equal(q.absmax_q.cpu().numpy(), ref["absmax_q"]), "u8 scales differ"
        assert q.absmax_scale.cpu().numpy()[0].view(np.uint32) == \
            np.float32(ref["absmax_scale"]).view(np.uint32)
    for out in ("f32", "bf16", "f16"):
        got = Q.dequantize(q, out).cpu()
        want = O.dequantize(ref, out)
        if out == "f32":
            assert np.array_equal(got.numpy().view(np.uint32), want.view(np.uint32)), out
        elif out == "bf16":
            assert np.array_equal(got.view(torch.int16).numpy().view(np.uint16), want), out
        else:
            assert np.array_equal(got.numpy().view(np.uint16), want.view(np.uint16)), out
    return q, ref


@pytest.mark.parametrize("rows,cols,bs", [
    (1, 100, 64),      # one whole block and a 36-element tail
    (7, 37, 64),       # odd element count: 4 whole blocks and a 3-element tail
    (1, 1, 64),        # a single element, no whole block
    (3, 333, 256),     # widest vectorized block, odd 231-element tail
    (5, 201, 8),       # narrowest vectorized block, 5-element tail
    (13, 77, 6),       # per-block path (6 is not a multiple of 8), odd count
    (11, 1001, 40),    # multiple of 8 but not a power of two, 11-element tail
    (3, 3, 2),         # smallest block, one-element tail
    (2, 1500, 1024),   # blocks wider than the kernel's 256 threads, 952-element tail
    (1, 700, 1024),    # no whole block; the tail spans three passes of the CTA
])
@pytest.mark.parametrize("dq", [False, True])
def test_short_last_block(cuda_device, rows, cols, bs, dq):
    w = WL.draw_weight((rows, cols), seed=4000 + rows * 7 + cols + bs)
    _check(w, bs, dq, cuda_device)


@pytest.mark.parametrize("kind", ["bf16", "f16"])
@pytest.mark.parametrize("rows,cols,bs", [(7, 37, 64), (13, 77, 6), (2, 1500, 1024)])
def test_short_last_block_typed_input(cuda_device, kind, rows, cols, bs):
    w = WL.draw_weight((rows, cols), seed=4100 + rows + cols + bs)
    _check(w, bs, True, cuda_device, kind)


def test_tail_holds_the_global_max(cuda_device):
    """The scale of scales comes from the short block alone."""
    w = WL.draw_weight((9, 71), seed=4201)
    w.reshape(-1)[-30:] *= np.float32(25.0)      # the last 639 - 576 = 63 elements hold the max
    q, ref = _check(w, 64, True, cuda_device)
    assert ref["absmax"].argmax() == ref["absmax"].size - 1


def test_zero_tail(cuda_device):
    """A short block of zeros: scale 0 and code 7 throughout."""
    w = WL.draw_weight((5, 27), seed=4202)
    w.reshape(-1)[128:] = 0.0
    q, ref = _check(w, 64, True, cuda_device)
    assert ref["absmax"][-1] == 0.0
    assert np.all(ref["codes"][64:] == 0x77)


def test_large_ragged_weight(cuda_device):
    """A 4095 x 4097 weight (16,777,215 elements: an odd 63-element tail)."""
    w = WL.draw_weight((4095, 4097), seed=4203)
    _check(w, 64, True, cuda_device)


def test_nonfinite_in_the_tail_is_flagged(cuda_device):
    import torch
    from qlora_linear_layers_nf4_b200 import nf4qlora as Q
    w = WL.draw_weight((3, 50), seed=4204)
    w[2, 49] = np.inf                               # element 149 of 150: in the 22-element tail
    ws = Q.Workspace(cuda_device)
    Q.quantize(torch.from_numpy(w).to(cuda_device), 64, True, workspace=ws)
    assert ws.read_status() == 7                    # NF4_ERR_NONFINITE
    Q.quantize(torch.from_numpy(w[:, :48].copy()).to(cuda_device), 64, True, workspace=ws)
    assert ws.read_status() == 0                    # the status was cleared by the read
