"""CPU checks of the C-ABI library: it loads, exports what the header
declares, reports the oracle's codebook, and refuses bad arguments on the host
before touching the GPU.  No compute call is made here."""
import ctypes
import os
import re
from fractions import Fraction

import numpy as np
import pytest

from oracle import nf4_oracle as O
from qlora_linear_layers_nf4_b200 import nf4qlora as Q
from tests.conftest import ROOT

FAKE = 0x10000   # aligned, never dereferenced: every call below fails validation first


def _declared():
    text = open(os.path.join(ROOT, "include", "nf4qlora.h")).read()
    return re.findall(r"NF4_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)


def test_library_exports_every_declared_symbol():
    L = Q.lib()
    names = _declared()
    assert set(names) == set(Q.EXPORTED)
    for n in names:
        assert hasattr(L, n), n


def test_codebook_matches_oracle_bit_for_bit():
    lv, th = Q.codebook()
    lv = np.array(lv, dtype=np.float32)
    assert np.array_equal(lv.view(np.uint32), O.nf4_levels().view(np.uint32))
    th = np.array(th, dtype=np.float32)
    for i in range(15):
        m = (Fraction(float(lv[i])) + Fraction(float(lv[i + 1]))) / 2
        nxt = np.nextafter(th[i], np.float32(2), dtype=np.float32)
        assert Fraction(float(th[i])) <= m < Fraction(float(nxt))


def test_threshold_count_rule_equals_oracle_nearest():
    # The library's encoding rule (count of thresholds below v) against the
    # oracle's brute-force nearest level, on midpoint neighbourhoods and randoms.
    _, th = Q.codebook()
    th = np.array(th, dtype=np.float32)
    rng = np.random.default_rng(1)
    v = np.concatenate([rng.uniform(-1, 1, 200000).astype(np.float32), th,
                        np.nextafter(th, np.float32(2)), np.nextafter(th, np.float32(-2)),
                        np.array([0.0, -0.0, 1.0, -1.0], np.float32)])
    count = (v[:, None] > th[None, :]).sum(axis=1)
    assert np.array_equal(count.astype(np.uint8), O.nearest_code(v))


def test_status_strings_and_version():
    L = Q.lib()
    for code, name in Q.STATUS_NAMES.items():
        assert L.nf4_status_string(code).decode().startswith(name)
    assert L.nf4_version() >= 100
    assert Q.launch_count() >= 0


def test_workspace_sizes():
    assert Q.workspace_bytes(Q.OP_DEQUANTIZE, 0, 4096, 4096, 0, 64, False) == 0
    assert Q.workspace_bytes(Q.OP_QUANTIZE, 0, 4096, 4096, 0, 64, False) >= 256
    assert Q.workspace_bytes(Q.OP_QUANTIZE, 0, 4096, 4096, 0, 64, True) >= 256 + 4096 * 64 * 4
    # a short last block is a block of its own: 3 blocks for 130 elements
    assert Q.workspace_bytes(Q.OP_QUANTIZE, 0, 13, 10, 0, 64, True) >= 256 + 3 * 4
    assert Q.workspace_bytes(Q.OP_LINEAR_FWD, 4096, 11008, 4096, 64, 64, True) >= 256
    assert Q.workspace_bytes(Q.OP_LINEAR_BWD, 4096, 11008, 4096, 64, 64, True) >= 256


def _quant(rows, cols, bs, dq, w=FAKE, codes=FAKE, absmax=FAKE, aq=FAKE, asc=FAKE, ws=FAKE, wsb=1 << 30):
    return Q.lib().nf4_quantize(w, rows, cols, bs, dq, codes, absmax, aq, asc, ws, wsb, None)


def test_quantize_host_validation():
    assert _quant(4, 64, 63, 0) == 2          # odd block size
    assert _quant(4, 64, 0, 0) == 2
    # a short last block (30 elements, block 64) passes the shape checks and
    # reaches the workspace check
    assert _quant(3, 10, 64, 1, wsb=16) == 5
    assert _quant(4, 64, 64, 2) == 1          # double_quant must be 0/1
    assert _quant(4, 64, 64, 0, w=None) == 1
    assert _quant(4, 64, 64, 0, absmax=None) == 1
    assert _quant(4, 64, 64, 1, aq=None) == 1
    assert _quant(4, 64, 64, 0, w=FAKE + 4) == 3
    assert _quant(4, 64, 64, 0, codes=FAKE + 8) == 3
    assert _quant(4, 64, 64, 0, ws=None) == 5
    assert _quant(4, 64, 64, 1, wsb=16) == 5
    assert _quant(-1, 64, 64, 0) == 2


def _cw(rows=4096, cols=4096, bs=64, dq=1, codes=FAKE):
    return Q.CWeight(codes=codes, absmax=FAKE, absmax_q=FAKE, absmax_scale=FAKE, rows=rows,
                     cols=cols, block_size=bs, double_quant=dq)


def test_dequantize_host_validation():
    L = Q.lib()
    assert L.nf4_dequantize(ctypes.byref(_cw(bs=7)), 0, FAKE, None) == 2        # odd block size
    assert L.nf4_dequantize(ctypes.byref(_cw(bs=0)), 0, FAKE, None) == 2
    # any even block size and a short last block pass the shape checks and
    # reach the alignment check of `out`
    assert L.nf4_dequantize(ctypes.byref(_cw(bs=6)), 0, FAKE + 2, None) == 3
    assert L.nf4_dequantize(ctypes.byref(_cw(rows=3, cols=8, bs=16)), 0, FAKE + 2, None) == 3
    assert L.nf4_dequantize(ctypes.byref(_cw()), 7, FAKE, None) == 1
    assert L.nf4_dequantize(ctypes.byref(_cw(codes=None)), 0, FAKE, None) == 1
    assert L.nf4_dequantize(ctypes.byref(_cw()), 0, FAKE + 2, None) == 3


def _fwd(cw, M=16, r=16, dtype=1, alpha=32.0, x=FAKE, y=FAKE, wsb=1 << 40):
    return Q.lib().qlora_linear_fwd(ctypes.byref(cw), x, M, FAKE, FAKE, r, alpha, dtype, None, y,
                                    None, FAKE, wsb, None)


def test_linear_host_validation():
    assert _fwd(_cw(), r=4) == 1                  # r < 8
    assert _fwd(_cw(), r=12) == 1                 # r % 8
    assert _fwd(_cw(), r=512) == 1
    assert _fwd(_cw(), dtype=2, wsb=0) == 5       # F16 compute passes the dtype check
    assert _fwd(_cw(), dtype=0, wsb=0) == 5       # F32 compute accepted: reaches the workspace check
    assert _fwd(_cw(), dtype=3) == 1              # no such dtype
    assert _fwd(_cw(), dtype=9) == 1
    assert _fwd(_cw(), M=0) == 2
    assert _fwd(_cw(cols=4000)) == 2              # K % 64
    assert _fwd(_cw(rows=4092)) == 2              # N % 8
    assert _fwd(_cw(bs=128), wsb=0) == 5          # powers of two from 64 to 4096 pass the checks
    assert _fwd(_cw(bs=4096), wsb=0) == 5
    assert _fwd(_cw(bs=32)) == 4                  # below 64: a K step would hold two blocks
    assert _fwd(_cw(bs=96)) == 4                  # not a power of two
    assert _fwd(_cw(bs=8192)) == 4
    assert _fwd(_cw(bs=0)) == 2
    assert _fwd(_cw(), x=FAKE + 2) == 3
    assert _fwd(_cw(), y=None) == 1
    assert _fwd(_cw(), wsb=0) == 5
    L = Q.lib()
    st = L.qlora_linear_bwd(ctypes.byref(_cw()), FAKE, 16, FAKE, FAKE, 16, 32.0, 1, None, None,
                            FAKE, FAKE, None, FAKE, 1 << 40, None)
    assert st == 1                                # dy required


def test_merge_host_validation():
    L = Q.lib()
    m = lambda cw, r=16, dt=1, out=FAKE, wsb=1 << 40: L.nf4_merge(
        ctypes.byref(cw), FAKE, FAKE, r, 32.0, dt, out, FAKE, wsb, None)
    assert m(_cw(), r=4) == 1                     # r < 8
    assert m(_cw(), r=264) == 1                   # r > 256
    assert m(_cw(), dt=2, wsb=0) == 5             # f16 output passes the dtype check
    assert m(_cw(), dt=7) == 1
    assert m(_cw(), out=None) == 1
    assert m(_cw(), out=FAKE + 2) == 3
    assert m(_cw(cols=4000)) == 2                 # K % 64
    assert m(_cw(bs=256), wsb=0) == 5             # powers of two from 64 to 4096
    assert m(_cw(bs=192)) == 4
    assert m(_cw(), wsb=0) == 5


def test_noalloc_host_validation():
    # nf4_quantize_noalloc checks its sizes against its fixed scratch array on
    # the host, before it looks the array up or launches anything.
    L = Q.lib()
    rows, cols = 16384, 4160          # 1,064,960 blocks of 64 > 1,048,576
    assert L.nf4_quantize_noalloc(FAKE, rows, cols, 64, 1, FAKE, None, FAKE, FAKE, None) == 5
    # with a caller absmax buffer the array holds no block scales: no size limit,
    # so the same size reaches the alignment check of `codes`
    assert L.nf4_quantize_noalloc(FAKE, rows, cols, 64, 1, FAKE + 8, FAKE, FAKE, FAKE, None) == 3
    assert L.nf4_quantize_noalloc(FAKE, 4, 64, 63, 0, FAKE, FAKE, None, None, None) == 2
    assert L.nf4_quantize_noalloc(FAKE, 4, 64, 64, 2, FAKE, FAKE, None, None, None) == 1
    assert L.nf4_quantize_noalloc(None, 4, 64, 64, 0, FAKE, FAKE, None, None, None) == 1
    assert L.nf4_quantize_noalloc(FAKE, 4, 64, 64, 0, FAKE, None, None, None, None) == 1
    assert L.nf4_quantize_noalloc(FAKE, 4, 64, 64, 1, FAKE, None, None, FAKE, None) == 1
    assert L.nf4_quantize_noalloc(FAKE + 4, 4, 64, 64, 0, FAKE, FAKE, None, None, None) == 3


def test_wait_check_host_validation():
    L = Q.lib()
    rel = ctypes.c_uint32(0)
    assert L.nf4_check_wait_timeout(None, 256, 1000, ctypes.byref(rel), None) == 5
    assert L.nf4_check_wait_timeout(FAKE, 16, 1000, ctypes.byref(rel), None) == 5
    assert L.nf4_check_wait_timeout(FAKE, 256, 0, ctypes.byref(rel), None) == 1
    assert L.nf4_check_wait_timeout(FAKE, 256, 2000000, ctypes.byref(rel), None) == 1
    assert L.nf4_check_wait_timeout(FAKE, 256, 1000, None, None) == 1


def test_bucket_encoding_conditions():
    # The quantize kernel's fast encode rounds 32 v + 32 to the nearest integer
    # i (one fused multiply-add, exact before its one rounding), so bucket i of
    # 65 covers [(i - 32.5) / 32, (i - 31.5) / 32) over v in [-1, 1], and
    # compares v with the single threshold that may lie inside the bucket.  It
    # is exact only if no bucket holds two thresholds and no threshold sits on
    # a bucket edge, where a tie could pick the neighbouring bucket.
    _, th = Q.codebook()
    th = np.array(th, dtype=np.float64)
    edges = (np.arange(66) - 32.5) / 32.0
    assert edges[0] < -1.0 and edges[-1] > 1.0
    assert np.min(np.abs(th[:, None] - edges[None, :])) > 2e-4
    counts = [np.sum((th >= edges[j]) & (th < edges[j + 1])) for j in range(65)]
    assert max(counts) <= 1
    assert sum(counts) == 15


def test_sharded_double_quant_host_validation():
    L = Q.lib()
    assert L.nf4_absmax_max(FAKE, -1, FAKE, None) == 2
    assert L.nf4_absmax_max(FAKE, 4, None, None) == 1
    assert L.nf4_absmax_max(None, 4, FAKE, None) == 1
    assert L.nf4_absmax_max(FAKE + 2, 4, FAKE, None) == 3
    assert L.nf4_double_quant(FAKE, -1, FAKE, FAKE, FAKE, None) == 2
    assert L.nf4_double_quant(FAKE, 4, None, FAKE, FAKE, None) == 1
    assert L.nf4_double_quant(FAKE, 4, FAKE, None, FAKE, None) == 1
    assert L.nf4_double_quant(FAKE, 4, FAKE, FAKE, None, None) == 1
    assert L.nf4_double_quant(FAKE + 4, 4, FAKE, FAKE, FAKE, None) == 3   # absmax 16-byte aligned
    assert L.nf4_double_quant(FAKE, 4, FAKE, FAKE + 4, FAKE, None) == 3


def _cpu_weight(rows=64, cols=128):
    import torch
    return Q.QuantizedWeight(codes=torch.zeros(rows * cols // 2, dtype=torch.uint8),
                             absmax=torch.zeros(rows * cols // 64, dtype=torch.float32),
                             absmax_q=None, absmax_scale=None, rows=rows, cols=cols,
                             block_size=64, double_quant=False)


def test_binding_refuses_mismatched_tensors():
    # Checked in the binding before anything reaches the C ABI (which sees
    # only pointers), so these run without a GPU.
    import torch
    q = _cpu_weight()
    bf, f16 = torch.bfloat16, torch.float16
    x = torch.zeros(8, 128, dtype=bf)
    A = torch.zeros(16, 128, dtype=bf)
    B = torch.zeros(64, 16, dtype=bf)
    with pytest.raises(TypeError):
        Q.linear_fwd(q, x, A.to(f16), B, 32.0)                  # A in another dtype than x
    with pytest.raises(ValueError):
        Q.linear_fwd(q, x, torch.zeros(16, 64, dtype=bf), B, 32.0)   # A's K is not the weight's
    with pytest.raises(ValueError):
        Q.linear_fwd(q, x, A, torch.zeros(32, 16, dtype=bf), 32.0)   # B's N is not the weight's
    with pytest.raises(ValueError):
        Q.linear_fwd(q, x, A, B.t().contiguous().t(), 32.0)          # not row-major
    with pytest.raises(ValueError):
        Q.linear_fwd(q, x, A, B, 32.0, bias=torch.zeros(63, dtype=bf))
    with pytest.raises(TypeError):
        Q.linear_fwd(q, x.to(torch.int32), A, B, 32.0)               # no such compute dtype
    dy = torch.zeros(8, 64, dtype=bf)
    with pytest.raises(ValueError):
        Q.linear_bwd(q, x, A, B, 32.0, torch.zeros(8, 63, dtype=bf))
    with pytest.raises(TypeError):
        Q.linear_bwd(q, x, A, B, 32.0, dy, dA=torch.zeros(16, 128, dtype=bf))   # dA is fp32
    with pytest.raises(ValueError):
        Q.linear_bwd(q, x, A, B, 32.0, dy, t=torch.zeros(8, 8, dtype=bf))
    with pytest.raises(TypeError):
        Q.merge(q, A.to(f16), B, 32.0)                               # merge adapters are bf16
    with pytest.raises(ValueError):
        Q.merge(q, A, B, 32.0, "bf16", out=torch.zeros(64, 64, dtype=bf))
