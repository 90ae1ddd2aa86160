"""GPU parity for row-sharded NF4 quantization with the simplified double
quant: nf4_absmax_max and nf4_double_quant, the two halves of the double
quant that a data-parallel quantization runs around its one exchange (an
all-reduce of the global max of the block scales).

On one GPU the shards of a weight are quantized one after another and the
all-reduce(MAX) is stood in for by the max of the shards' results; the
shards' codes and u8 scales, put together, must be bit for bit the oracle's
(and the library's own) quantization of the whole weight.
"""
import numpy as np
import pytest

from oracle import nf4_oracle as O
from qlora_linear_layers_nf4_b200 import workloads as WL

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("rows,cols,nshards", [(256, 512, 2), (4096, 4096, 4), (96, 200, 3)])
def test_sharded_double_quant_matches_whole(cuda_device, rows, cols, nshards):
    import torch
    from qlora_linear_layers_nf4_b200 import nf4qlora as Q
    w = WL.draw_weight((rows, cols), seed=9000 + rows + nshards)
    w[-(rows // nshards):] *= np.float32(4.0)          # the global max sits in the last shard
    whole = O.quantize(w, 64, double=True)
    per = rows // nshards
    shards = [torch.from_numpy(np.ascontiguousarray(w[i * per:(i + 1) * per])).to(cuda_device)
              for i in range(nshards)]
    qs = [Q.quantize(s, 64, False, keep_absmax=True) for s in shards]
    local = [Q.absmax_max(q.absmax) for q in qs]
    g = torch.stack(local).max().reshape(1)           # stands in for all_reduce(MAX)
    dq = [Q.double_quant(q.absmax, g) for q in qs]
    torch.cuda.synchronize()
    for q, gl in zip(qs, local):
        assert gl.item() == float(q.absmax.max())
    assert np.float32(g.item()) == np.float32(whole["absmax"].max())
    codes = np.concatenate([q.codes.cpu().numpy() for q in qs])
    aq = np.concatenate([a.cpu().numpy() for a, _ in dq])
    assert np.array_equal(codes, whole["codes"])
    assert np.array_equal(aq, whole["absmax_q"])
    for _, s in dq:
        assert s.cpu().numpy()[0].view(np.uint32) == np.float32(whole["absmax_scale"]).view(np.uint32)
    # the library's single-call double quant gives the same
    full = Q.quantize(torch.from_numpy(w).to(cuda_device), 64, True)
    assert np.array_equal(full.absmax_q.cpu().numpy(), aq)


def test_quantize_sharded_one_rank_is_quantize(cuda_device):
    import torch
    from qlora_linear_layers_nf4_b200 import dp
    from qlora_linear_layers_nf4_b200 import nf4qlora as Q
    w = torch.from_numpy(WL.draw_weight((512, 1024), seed=9100)).to(cuda_device)
    qs = dp.quantize_sharded(w, 64, True)
    ref = Q.quantize(w, 64, True)
    torch.cuda.synchronize()
    assert torch.equal(qs.codes, ref.codes)
    assert torch.equal(qs.absmax_q, ref.absmax_q)
    assert torch.equal(qs.absmax_scale.view(torch.int32), ref.absmax_scale.view(torch.int32))
    # and it decodes like the library's own double-quantized weight
    assert torch.equal(Q.dequantize(qs, "f32").view(torch.int32), Q.dequantize(ref, "f32").view(torch.int32))


def test_absmax_max_edges(cuda_device):
    import torch
    from qlora_linear_layers_nf4_b200 import nf4qlora as Q
    empty = torch.empty(0, dtype=torch.float32, device=cuda_device)
    assert Q.absmax_max(empty).item() == 0.0
    a = torch.zeros(1000, dtype=torch.float32, device=cuda_device)
    assert Q.absmax_max(a).item() == 0.0
    a[777] = 3.5
    assert Q.absmax_max(a).item() == 3.5
    aq, s = Q.double_quant(torch.zeros(5, dtype=torch.float32, device=cuda_device),
                           torch.zeros(1, dtype=torch.float32, device=cuda_device))
    assert s.item() == 0.0 and int(aq.max()) == 0
