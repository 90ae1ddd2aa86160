"""GPU parity: NF4 quantize of bf16 and f16 weights (nf4_quantize_typed), bit
for bit against the CPU oracle quantizing the same values widened to fp32
(the widening is exact, so that is the whole definition)."""
import numpy as np
import pytest

from oracle import nf4_oracle as O
from qlora_linear_layers_nf4_b200 import workloads as WL

pytestmark = pytest.mark.gpu


def _as_input(w32, kind):
    """(numpy values the oracle sees, torch tensor the GPU quantizes)."""
    import torch
    if kind == "bf16":
        bits = WL.to_bf16_bits(w32)
        t = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)
        return WL.bf16_bits_to_f32(bits).reshape(w32.shape), t.reshape(w32.shape)
    h = w32.astype(np.float16)
    return h.astype(np.float32), torch.from_numpy(h)


def _check(w32, kind, bs, dq, dev):
    import torch
    from qlora_linear_layers_nf4_b200 import nf4qlora as Q
    vals, t = _as_input(w32, kind)
    ref = O.quantize(vals, bs, double=dq)
    q = Q.quantize(t.to(dev), bs, dq, keep_absmax=True, check_status=True)
    torch.cuda.synchronize()
    assert np.array_equal(q.codes.cpu().numpy()[: ref["codes"].size], ref["codes"])
    assert np.array_equal(q.absmax.cpu().numpy()[: ref["absmax"].size].view(np.uint32),
                          ref["absmax"].view(np.uint32))
    if dq:
        assert np.array_equal(q.absmax_q.cpu().numpy()[: ref["absmax_q"].size], ref["absmax_q"])
        assert q.absmax_scale.cpu().numpy()[0].view(np.uint32) == np.float32(ref["absmax_scale"]).view(np.uint32)


@pytest.mark.parametrize("kind", ["bf16", "f16"])
@pytest.mark.parametrize("bs,dq", [(64, True), (64, False), (32, True), (128, False), (40, True)])
def test_typed_block_sizes(cuda_device, kind, bs, dq):
    w = WL.draw_weight((13, bs * 29), seed=500 + bs)
    _check(w, kind, bs, dq, cuda_device)


@pytest.mark.parametrize("kind", ["bf16", "f16"])
def test_typed_full_4096_square(cuda_device, kind):
    w = WL.draw_weight(WL.QUANT_SHAPE, WL.QUANT_SEED)
    _check(w, kind, 64, True, cuda_device)


def test_typed_nonfinite_is_flagged(cuda_device):
    import torch
    from qlora_linear_layers_nf4_b200 import nf4qlora as Q
    w = WL.draw_weight((8, 64), seed=9)
    t = torch.from_numpy(w).to(torch.bfloat16)
    t[2, 7] = float("inf")
    ws = Q.Workspace(cuda_device)
    Q.quantize(t.to(cuda_device), 64, True, workspace=ws)
    assert ws.read_status() == 7
