"""Thin ctypes binding of libnf4qlora.so (declared in include/nf4qlora.h).

Argument marshalling only: every step of the computation runs in the CUDA
library.  PyTorch provides device memory (and the workspace) and the current
stream.  There is no fallback: if the library is missing or the GPU call
fails, these functions raise.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libnf4qlora.so")

NF4_OK = 0
STATUS_NAMES = {
    0: "NF4_OK", 1: "NF4_ERR_INVALID_ARG", 2: "NF4_ERR_SHAPE", 3: "NF4_ERR_ALIGNMENT",
    4: "NF4_ERR_UNSUPPORTED", 5: "NF4_ERR_WORKSPACE", 6: "NF4_ERR_CUDA",
    7: "NF4_ERR_NONFINITE", 8: "NF4_ERR_TIMEOUT",
}
NF4_F32, NF4_BF16, NF4_F16 = 0, 1, 2
OP_QUANTIZE, OP_DEQUANTIZE, OP_LINEAR_FWD, OP_LINEAR_BWD, OP_MERGE = 0, 1, 2, 3, 4

EXPORTED = (
    "nf4_status_string", "nf4_version", "nf4_codebook", "nf4_launch_count",
    "nf4_profile_begin", "nf4_profile_end", "nf4_profile_kernel_count", "nf4_kernel_name",
    "nf4_profile_get", "nf4_workspace_bytes", "nf4_read_status", "nf4_quantize",
    "nf4_dequantize", "qlora_linear_fwd", "qlora_linear_bwd", "nf4_quantize_noalloc",
    "nf4_merge", "nf4_quantize_typed", "nf4_check_wait_timeout", "nf4_absmax_max",
    "nf4_double_quant",
)


class NF4Error(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = int(status)
        name = STATUS_NAMES.get(self.status, str(status))
        super().__init__(f"{what}: {name}" if what else name)


class CWeight(ctypes.Structure):
    """Mirror of `nf4_weight`."""
    _fields_ = [
        ("codes", ctypes.c_void_p),
        ("absmax", ctypes.c_void_p),
        ("absmax_q", ctypes.c_void_p),
        ("absmax_scale", ctypes.c_void_p),
        ("rows", ctypes.c_int64),
        ("cols", ctypes.c_int64),
        ("block_size", ctypes.c_int32),
        ("double_quant", ctypes.c_int32),
    ]


_lib = None


def lib() -> ctypes.CDLL:
    """Load the library once; raise if it was not built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m qlora_linear_layers_nf4_b200.build` "
            "(there is no CPU fallback)")
    L = ctypes.CDLL(LIB_PATH)
    vp, i64, i32, f32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    L.nf4_status_string.argtypes = [i32]
    L.nf4_status_string.restype = ctypes.c_char_p
    L.nf4_version.restype = i32
    L.nf4_codebook.argtypes = [vp, vp]
    L.nf4_codebook.restype = None
    L.nf4_launch_count.restype = i64
    L.nf4_profile_begin.restype = i32
    L.nf4_profile_end.restype = i32
    L.nf4_profile_kernel_count.restype = i32
    L.nf4_kernel_name.argtypes = [i32]
    L.nf4_kernel_name.restype = ctypes.c_char_p
    L.nf4_profile_get.argtypes = [i32, ctypes.POINTER(i64), ctypes.POINTER(ctypes.c_double)]
    L.nf4_profile_get.restype = i32
    L.nf4_workspace_bytes.argtypes = [i32, i64, i64, i64, i32, i32, i32]
    L.nf4_workspace_bytes.restype = sz
    L.nf4_read_status.argtypes = [vp, vp]
    L.nf4_read_status.restype = i32
    L.nf4_quantize.argtypes = [vp, i64, i64, i32, i32, vp, vp, vp, vp, vp, sz, vp]
    L.nf4_quantize.restype = i32
    L.nf4_quantize_noalloc.argtypes = [vp, i64, i64, i32, i32, vp, vp, vp, vp, vp]
    L.nf4_quantize_noalloc.restype = i32
    L.nf4_dequantize.argtypes = [ctypes.POINTER(CWeight), i32, vp, vp]
    L.nf4_dequantize.restype = i32
    L.qlora_linear_fwd.argtypes = [ctypes.POINTER(CWeight), vp, i64, vp, vp, i32, f32, i32, vp, vp,
                                   vp, vp, sz, vp]
    L.qlora_linear_fwd.restype = i32
    L.qlora_linear_bwd.argtypes = [ctypes.POINTER(CWeight), vp, i64, vp, vp, i32, f32, i32, vp, vp,
                                   vp, vp, vp, vp, sz, vp]
    L.qlora_linear_bwd.restype = i32
    L.nf4_merge.argtypes = [ctypes.POINTER(CWeight), vp, vp, i32, f32, i32, vp, vp, sz, vp]
    L.nf4_merge.restype = i32
    L.nf4_quantize_typed.argtypes = [vp, i32, i64, i64, i32, i32, vp, vp, vp, vp, vp, sz, vp]
    L.nf4_quantize_typed.restype = i32
    L.nf4_check_wait_timeout.argtypes = [vp, sz, ctypes.c_uint32, ctypes.POINTER(ctypes.c_uint32), vp]
    L.nf4_check_wait_timeout.restype = i32
    L.nf4_absmax_max.argtypes = [vp, i64, vp, vp]
    L.nf4_absmax_max.restype = i32
    L.nf4_double_quant.argtypes = [vp, i64, vp, vp, vp, vp]
    L.nf4_double_quant.restype = i32
    _lib = L
    return L


def _check(status: int, what: str):
    if status != NF4_OK:
        raise NF4Error(status, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def codebook():
    """(levels[16], thresholds[15]) as Python float lists, from the library."""
    lv = (ctypes.c_float * 16)()
    th = (ctypes.c_float * 15)()
    lib().nf4_codebook(ctypes.cast(lv, ctypes.c_void_p), ctypes.cast(th, ctypes.c_void_p))
    return list(lv), list(th)


def launch_count() -> int:
    return int(lib().nf4_launch_count())


def profile_begin():
    _check(lib().nf4_profile_begin(), "nf4_profile_begin")


def profile_end() -> dict:
    """Stop recording; {kernel name: (timed launches, total ms)} for kernels that ran."""
    _check(lib().nf4_profile_end(), "nf4_profile_end")
    out = {}
    L = lib()
    for i in range(L.nf4_profile_kernel_count()):
        n = ctypes.c_int64()
        ms = ctypes.c_double()
        _check(L.nf4_profile_get(i, ctypes.byref(n), ctypes.byref(ms)), "nf4_profile_get")
        if n.value:
            out[L.nf4_kernel_name(i).decode()] = (int(n.value), float(ms.value))
    return out


def workspace_bytes(op: int, M: int, N: int, K: int, r: int, block_size: int, double_quant: bool) -> int:
    return int(lib().nf4_workspace_bytes(op, M, N, K, r, block_size, int(double_quant)))


class Workspace:
    """A zero-filled device byte buffer reused across calls (grown on demand)."""

    def __init__(self, device=None):
        self.device = device
        self.buf = None

    def get(self, nbytes: int):
        import torch
        nbytes = max(int(nbytes), 256)
        if self.buf is None or self.buf.numel() < nbytes:
            dev = self.device if self.device is not None else torch.device("cuda", torch.cuda.current_device())
            self.buf = torch.zeros(nbytes, dtype=torch.uint8, device=dev)
        return self.buf

    def read_status(self, stream=None) -> int:
        if self.buf is None:
            return NF4_OK
        return int(lib().nf4_read_status(_ptr(self.buf), _stream(stream)))


_default_ws = {}


def default_workspace(device) -> Workspace:
    key = str(device)
    if key not in _default_ws:
        _default_ws[key] = Workspace(device)
    return _default_ws[key]


@dataclass
class QuantizedWeight:
    """Device tensors of one NF4 weight (fields as in `nf4_weight`)."""
    codes: object                    # uint8 [ceil(numel/2)]
    absmax: object | None            # fp32 [nblocks = ceil(numel/block_size)]
    absmax_q: object | None          # uint8 [nblocks]
    absmax_scale: object | None      # fp32 [1]
    rows: int
    cols: int
    block_size: int
    double_quant: bool

    def c_struct(self) -> CWeight:
        return CWeight(
            codes=self.codes.data_ptr(),
            absmax=None if (self.absmax is None or self.double_quant) else self.absmax.data_ptr(),
            absmax_q=None if self.absmax_q is None else self.absmax_q.data_ptr(),
            absmax_scale=None if self.absmax_scale is None else self.absmax_scale.data_ptr(),
            rows=self.rows, cols=self.cols, block_size=self.block_size,
            double_quant=int(self.double_quant))

    @property
    def device(self):
        return self.codes.device


def quantize(w, block_size: int = 64, double_quant: bool = False, keep_absmax: bool | None = None,
             workspace: Workspace | None = None, stream=None, check_status: bool = False) -> QuantizedWeight:
    """NF4-quantize a float32, bfloat16 or float16 CUDA tensor (any shape;
    flattened row-major).  bf16 / f16 elements are widened to fp32 exactly."""
    import torch
    in_dtype = {torch.float32: NF4_F32, torch.bfloat16: NF4_BF16, torch.float16: NF4_F16}.get(w.dtype)
    if in_dtype is None or not w.is_cuda:
        raise TypeError("quantize expects a float32, bfloat16 or float16 CUDA tensor")
    w = w.contiguous()
    rows = int(w.shape[0]) if w.dim() >= 1 else 1
    cols = 1
    for d in w.shape[1:]:
        cols *= int(d)
    numel = w.numel()
    dev = w.device
    nblocks = -(-numel // block_size) if block_size > 0 else 0   # the last block may be short
    keep_absmax = (not double_quant) if keep_absmax is None else keep_absmax
    codes = torch.empty(max((numel + 1) // 2, 1), dtype=torch.uint8, device=dev)
    absmax = torch.empty(max(nblocks, 1), dtype=torch.float32, device=dev) if keep_absmax else None
    absmax_q = torch.empty(max(nblocks, 1), dtype=torch.uint8, device=dev) if double_quant else None
    absmax_scale = torch.empty(1, dtype=torch.float32, device=dev) if double_quant else None
    ws = workspace or default_workspace(dev)
    buf = ws.get(workspace_bytes(OP_QUANTIZE, 0, rows, cols, 0, block_size, double_quant))
    if in_dtype == NF4_F32:
        st = lib().nf4_quantize(_ptr(w), rows, cols, block_size, int(double_quant), _ptr(codes),
                                _ptr(absmax), _ptr(absmax_q), _ptr(absmax_scale), _ptr(buf),
                                buf.numel(), _stream(stream))
    else:
        st = lib().nf4_quantize_typed(_ptr(w), in_dtype, rows, cols, block_size, int(double_quant),
                                      _ptr(codes), _ptr(absmax), _ptr(absmax_q), _ptr(absmax_scale),
                                      _ptr(buf), buf.numel(), _stream(stream))
    _check(st, "nf4_quantize")
    if check_status:
        _check(ws.read_status(stream), "nf4_quantize (device)")
    return QuantizedWeight(codes, absmax, absmax_q, absmax_scale, rows, cols, block_size, double_quant)


def absmax_max(absmax, stream=None):
    """Max of a CUDA fp32 tensor of block scales, as a 1-element CUDA tensor."""
    import torch
    g = torch.empty(1, dtype=torch.float32, device=absmax.device)
    _check(lib().nf4_absmax_max(_ptr(absmax), absmax.numel(), _ptr(g), _stream(stream)), "nf4_absmax_max")
    return g


def double_quant(absmax, gmax, stream=None):
    """The double-quant stage against a given global max (1-element CUDA
    tensor): returns (absmax_q uint8 [n], absmax_scale fp32 [1])."""
    import torch
    n = absmax.numel()
    aq = torch.empty(max(n, 1), dtype=torch.uint8, device=absmax.device)
    asc = torch.empty(1, dtype=torch.float32, device=absmax.device)
    _check(lib().nf4_double_quant(_ptr(absmax), n, _ptr(gmax), _ptr(aq), _ptr(asc), _stream(stream)),
           "nf4_double_quant")
    return aq, asc


def dequantize(q: QuantizedWeight, out_dtype: str = "f32", stream=None):
    import torch
    dt = {"f32": (NF4_F32, torch.float32), "bf16": (NF4_BF16, torch.bfloat16),
          "f16": (NF4_F16, torch.float16)}[out_dtype]
    out = torch.empty((q.rows, q.cols), dtype=dt[1], device=q.device)
    cw = q.c_struct()
    _check(lib().nf4_dequantize(ctypes.byref(cw), dt[0], _ptr(out), _stream(stream)), "nf4_dequantize")
    return out


def merge(q: QuantizedWeight, A, B, alpha: float, out_dtype: str = "bf16", out=None,
          workspace: Workspace | None = None, stream=None):
    """Dense merged weight dequant(W) + (alpha/r) B A, [rows, cols] in bf16, f16 or f32."""
    import torch
    dt = {"f32": (NF4_F32, torch.float32), "bf16": (NF4_BF16, torch.bfloat16),
          "f16": (NF4_F16, torch.float16)}[out_dtype]
    if A.dim() != 2:
        raise ValueError("A must be 2-D ([r, K])")
    r = A.shape[0]
    dev = q.device
    _expect("A", A, (r, q.cols), torch.bfloat16, dev)
    _expect("B", B, (q.rows, r), torch.bfloat16, dev)
    _expect("out", out, (q.rows, q.cols), dt[1], dev)
    if out is None:
        out = torch.empty((q.rows, q.cols), dtype=dt[1], device=q.device)
    ws = workspace if workspace is not None else Workspace(q.device)
    need = lib().nf4_workspace_bytes(OP_MERGE, 0, q.rows, q.cols, r, q.block_size, int(q.double_quant))
    buf = ws.get(need)
    cw = q.c_struct()
    _check(lib().nf4_merge(ctypes.byref(cw), _ptr(A), _ptr(B), r, float(alpha), dt[0], _ptr(out),
                           _ptr(buf), buf.numel(), _stream(stream)), "nf4_merge")
    return out


def _compute_dtype(x):
    """The C ABI's compute type for activations of x's dtype: bf16, f16, or
    fp32 (the CUDA-core fp32 reference mode)."""
    import torch
    if x.dtype == torch.bfloat16:
        return NF4_BF16
    if x.dtype == torch.float16:
        return NF4_F16
    if x.dtype == torch.float32:
        return NF4_F32
    raise TypeError(f"compute dtype must be bfloat16, float16 or float32, got {x.dtype}")


def _expect(name: str, t, shape, dtype, device):
    """The C ABI sees only a pointer: a tensor of the wrong shape, dtype,
    layout or device would be read as garbage, so the binding refuses it."""
    if t is None:
        return
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if t.dtype != dtype:
        raise TypeError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous (row-major)")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, the weight on {device}")


def _linear_shapes(q: QuantizedWeight, x, A):
    if x.dim() != 2 or A.dim() != 2:
        raise ValueError("x and A must be 2-D ([M, K] and [r, K])")
    return int(x.shape[0]), int(A.shape[0]), q.rows, q.cols


def linear_fwd(q: QuantizedWeight, x, A, B, alpha: float, bias=None, want_t: bool = True,
               out=None, t_out=None, workspace: Workspace | None = None, stream=None):
    """y = x W'^T + (alpha/r) (x A^T) B^T (+ bias); returns (y, T or None).

    x, A, B (and bias) share one compute dtype, bfloat16, float16 or float32
    (the fp32 reference mode); y and T come back in it."""
    import torch
    dt = _compute_dtype(x)
    M, r, N, K = _linear_shapes(q, x, A)
    dev = q.device
    _expect("x", x, (M, K), x.dtype, dev)
    _expect("A", A, (r, K), x.dtype, dev)
    _expect("B", B, (N, r), x.dtype, dev)
    _expect("bias", bias, (N,), x.dtype, dev)
    _expect("out", out, (M, N), x.dtype, dev)
    _expect("t_out", t_out, (M, r), x.dtype, dev)
    y = out if out is not None else torch.empty((M, q.rows), dtype=x.dtype, device=x.device)
    if want_t and t_out is None:
        t_out = torch.empty((M, r), dtype=x.dtype, device=x.device)
    ws = workspace or default_workspace(x.device)
    buf = ws.get(workspace_bytes(OP_LINEAR_FWD, M, q.rows, q.cols, r, q.block_size, q.double_quant))
    cw = q.c_struct()
    st = lib().qlora_linear_fwd(ctypes.byref(cw), _ptr(x), M, _ptr(A), _ptr(B), r, float(alpha),
                                dt, _ptr(bias), _ptr(y), _ptr(t_out), _ptr(buf), buf.numel(),
                                _stream(stream))
    _check(st, "qlora_linear_fwd")
    return y, t_out


def linear_bwd(q: QuantizedWeight, x, A, B, alpha: float, dy, t=None, want_dx: bool = True,
               dA=None, dB=None, dx=None, workspace: Workspace | None = None, stream=None):
    """Adapter backward; returns (dA fp32 [r,K], dB fp32 [N,r], dx [M,K] in x's dtype or None)."""
    import torch
    dt = _compute_dtype(x)
    M, r, N, K = _linear_shapes(q, x, A)
    dev = q.device
    _expect("x", x, (M, K), x.dtype, dev)
    _expect("A", A, (r, K), x.dtype, dev)
    _expect("B", B, (N, r), x.dtype, dev)
    _expect("dy", dy, (M, N), x.dtype, dev)
    _expect("t", t, (M, r), x.dtype, dev)
    _expect("dA", dA, (r, K), torch.float32, dev)
    _expect("dB", dB, (N, r), torch.float32, dev)
    _expect("dx", dx, (M, K), x.dtype, dev)
    dA = dA if dA is not None else torch.empty((r, q.cols), dtype=torch.float32, device=x.device)
    dB = dB if dB is not None else torch.empty((q.rows, r), dtype=torch.float32, device=x.device)
    if want_dx and dx is None:
        dx = torch.empty((M, q.cols), dtype=x.dtype, device=x.device)
    ws = workspace or default_workspace(x.device)
    buf = ws.get(workspace_bytes(OP_LINEAR_BWD, M, q.rows, q.cols, r, q.block_size, q.double_quant))
    cw = q.c_struct()
    st = lib().qlora_linear_bwd(ctypes.byref(cw), _ptr(x), M, _ptr(A), _ptr(B), r, float(alpha),
                                dt, _ptr(dy), _ptr(t), _ptr(dA), _ptr(dB), _ptr(dx),
                                _ptr(buf), buf.numel(), _stream(stream))
    _check(st, "qlora_linear_bwd")
    return dA, dB, dx
