"""GPU test of nf4_quantize_noalloc, the quantize entry point for callers
that cannot allocate device memory (no workspace argument; its scratch is a
fixed array inside the library).

It must give exactly what nf4_quantize gives.  Two calls in a row on
different weights check that the shared array's leftover contents (the
previous call's global max) do not leak into the next call.  This file is
collected last so a failure here cannot hide the other tests."""
import ctypes

import numpy as np
import pytest

from qlora_linear_layers_nf4_b200 import workloads as WL

pytestmark = pytest.mark.gpu


def _noalloc(L, w, bs, dq, use_own_absmax):
    import torch
    numel = w.numel()
    nb = -(-numel // bs)                  # the last block may be short
    dev = w.device
    codes = torch.empty((numel + 1) // 2, dtype=torch.uint8, device=dev)
    absmax = torch.empty(nb, dtype=torch.float32, device=dev) if (use_own_absmax or not dq) else None
    aq = torch.empty(nb, dtype=torch.uint8, device=dev) if dq else None
    asc = torch.empty(1, dtype=torch.float32, device=dev) if dq else None
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    st = L.nf4_quantize_noalloc(p(w), w.shape[0], w.shape[1], bs, int(dq), p(codes), p(absmax),
                                p(aq), p(asc), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, f"nf4_quantize_noalloc returned {st}"
    return codes, absmax, aq, asc


def test_noalloc_matches_quantize_two_calls(cuda_device):
    import torch
    from qlora_linear_layers_nf4_b200 import nf4qlora as Q
    L = Q.lib()
    weights = [WL.draw_weight((4096, 4096), seed=1, sigma=0.02),      # the 4096x4096 matrix
               WL.draw_weight((768, 1024), seed=5, sigma=0.005),      # smaller max: stale max would show
               WL.draw_weight((97, 45), seed=6, sigma=0.001)]         # a short, odd-sized last block
    for call, wn in enumerate(weights):
        w = torch.from_numpy(wn).to(cuda_device)
        for dq, own in ((True, False), (True, True), (False, True)):
            ref = Q.quantize(w, 64, dq, keep_absmax=True)
            before = Q.launch_count()
            codes, absmax, aq, asc = _noalloc(L, w, 64, dq, own)
            assert Q.launch_count() - before >= (2 if dq else 1), "launches not counted"
            torch.cuda.synchronize()
            assert torch.equal(codes, ref.codes), f"call {call}: codes differ"
            if absmax is not None:
                assert torch.equal(absmax.view(torch.int32), ref.absmax.view(torch.int32))
            if dq:
                assert torch.equal(aq, ref.absmax_q), f"call {call}: u8 scales differ"
                assert torch.equal(asc.view(torch.int32), ref.absmax_scale.view(torch.int32))

