"""The bounded-wait path, exercised on purpose and without any GPU fault: a
wait on an mbarrier that nothing arrives on gives up after its limit, records
NF4_ERR_TIMEOUT, and its abort flag releases the CTA's other waiting role;
the context stays usable afterwards."""
import ctypes
import time

import numpy as np
import pytest

from oracle import nf4_oracle as O
from qlora_linear_layers_nf4_b200 import workloads as WL

pytestmark = pytest.mark.gpu


def test_wait_gives_up_reports_and_releases(cuda_device):
    import torch
    from qlora_linear_layers_nf4_b200 import nf4qlora as Q
    L = Q.lib()
    ws = Q.Workspace(cuda_device)
    buf = ws.get(256)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    released = ctypes.c_uint32(0)
    t0 = time.perf_counter()
    st = L.nf4_check_wait_timeout(ctypes.c_void_p(buf.data_ptr()), buf.numel(), 20000,
                                  ctypes.byref(released), stream)
    elapsed = time.perf_counter() - t0
    assert st == 8, Q.status_name(st) if hasattr(Q, "status_name") else st   # NF4_ERR_TIMEOUT
    assert released.value == 2            # both CTAs' second role left on the abort flag
    assert elapsed < 1.0                  # not the 2 s of the second role's own limit
    assert ws.read_status() == 0          # the call cleared the word it reported
    # the context is still usable: a quantize right after is bit-exact
    w = WL.draw_weight((16, 128), seed=21)
    q = Q.quantize(torch.from_numpy(w).to(cuda_device), 64, True, workspace=ws)
    torch.cuda.synchronize()
    ref = O.quantize(w, 64, double=True)
    assert np.array_equal(q.codes.cpu().numpy(), ref["codes"])
    assert ws.read_status() == 0
