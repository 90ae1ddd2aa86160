"""CPU oracle for blockwise NF4 quantization and the QLoRA linear layer.

TEST INFRASTRUCTURE ONLY.  This module is the plain, slow, obviously correct
statement of what the CUDA library computes.  Only the test suite, the smoke
check and the benchmark's CPU-baseline leg may import it; the product path
(the C-ABI library and its Python binding) never does, and this module never
imports the product.  It shares no code, table or constant with the CUDA
sources: the sixteen NF4 levels are derived here from the normal quantile
function, not copied from the library.

Sources (web pages on the subject; each function names the passage it
follows):
  [P1] qlora-rs README (github, tzervas/qlora-rs): sections "Honest
       capability matrix", "Quick Start", "NF4 Quantization",
       "Double quantization (simplified)".
  [P2] rust-ai-core docs, struct QLoraConfig: sections "Compute Dtype",
       "Implementations" (scale() = alpha / r).
  [P3] qlora-rs 1.0.5 source page src/export.rs: the QuantizedTensor fields
       (data, scales, scales_quantized, scales_scales, shape), the
       merge_and_export_gguf docstring (W_merged = W_base + (B @ A) * scale)
       and its unit tests (an all-zeros tensor must quantize).
  [P4] "LoRA and QLoRA, mathematically": sections "The low-rank update
       hypothesis" (W0 in R^{d x k}), "Rank, alpha, and target modules"
       (alpha/r scaling), "NF4: quantizing the frozen base" (levels at normal
       quantiles, equally likely), "The merge math" (equation 6.3.6).

Readings of points the pages leave open:
  R1  NF4 construction: the pages print the levels to three decimals and say
      they sit at normal quantiles; the formula itself (equations 6.3.4-6.3.5)
      did not survive.  Reading: 8 positive quantiles
      Phi^-1(delta + (0.5 - delta) i / 8), i = 0..7, 7 negative ones
      -Phi^-1(delta + (0.5 - delta) i / 7), i = 0..6, plus an exact 0, divided
      by the largest magnitude, with delta = 1 - (1/32 + 1/30) / 2.  This is
      the QLoRA construction and the only simple delta that reproduces the
      printed table.
  R2  Blocks are consecutive elements of the row-major flattened tensor.
  R3  absmax == 0: every code is 7 (the exact zero level), absmax stored as 0.
  R4  v = fp32(w / absmax) with IEEE division; code = nearest level in exact
      arithmetic; an exact tie goes to the lower code.
  R5  Packing: byte j = code[2j] << 4 | code[2j+1] (first element in the high
      nibble).
  R6  Double quant: G = max absmax, s_g = fp32(G / 255),
      q = clip(rint_half_even(fp32(absmax / s_g)), 0, 255); G == 0 gives
      s_g = 0 and q = 0.  Dequantized scale = fp32(float(q) * s_g).
  R7  Dequant: w' = fp32(L[code] * scale); bf16 output is the round-to-nearest-
      even of that fp32 value, f16 likewise.
  R8  QLoRA forward in BF16 compute: y = x W'^T + s (x A^T) B^T (+ bias) with
      W' = bf16(dequant), s = alpha / r, evaluated here in fp64 from the exact
      bf16 inputs.
  R9  Backward of L = sum(dy * y) with W frozen: dB = s dy^T (x A^T),
      dA = s (dy B)^T x, dx = dy W' + s (dy B) A.
  R16 Merge: W_merged = w' + s B A from the fp32 dequant w' (not the bf16
      one), the sum taken exactly and rounded to fp32, then (for a bf16
      result) to bf16 with ties to even.
  R19 A tensor whose size is not a multiple of the block: the last block holds
      the remaining elements and its absmax is theirs alone; for an odd
      element count the last byte's low nibble is 7 (the exact-zero level).
  R20 F32 compute (listed as honoured, called the debugging mode): the base
      is the fp32 dequant w' itself, not rounded further; the forward and
      backward below are evaluated in fp64 from it and the fp32 inputs.
"""
from __future__ import annotations

from statistics import NormalDist

import numpy as np

__all__ = [
    "nf4_levels_f64",
    "nf4_levels",
    "nearest_code",
    "pack_codes",
    "unpack_codes",
    "quantize",
    "double_quant",
    "block_scales",
    "dequantize",
    "bf16_round",
    "bf16_to_f32",
    "qlora_forward",
    "qlora_backward",
    "merge",
    "matmul_bruteforce",
]

# ---------------------------------------------------------------------------
# NF4 levels  ([P4] "NF4: quantizing the frozen base"; [P1] "NF4 Quantization")
# ---------------------------------------------------------------------------

def nf4_levels_f64() -> np.ndarray:
    """The sixteen NF4 levels in fp64, ascending (reading R1).

    Levels sit at quantiles of the standard normal so that each is equally
    likely under a Gaussian source ([P4]); there is an exact zero and the
    endpoints are -1 and +1 after normalising by the largest magnitude ([P1]
    prints -1.0 ... 0.0 ... 1.0).
    """
    phi_inv = NormalDist().inv_cdf
    delta = 1.0 - 0.5 * (1.0 / 32.0 + 1.0 / 30.0)
    positive = [phi_inv(delta + (0.5 - delta) * i / 8.0) for i in range(8)]
    negative = [-phi_inv(delta + (0.5 - delta) * i / 7.0) for i in range(7)]
    levels = sorted(positive + negative + [0.0])
    biggest = max(abs(v) for v in levels)
    return np.array([v / biggest for v in levels], dtype=np.float64)


def nf4_levels() -> np.ndarray:
    """The NF4 codebook as fp32 (each fp64 level rounded to nearest)."""
    return nf4_levels_f64().astype(np.float32)


# ---------------------------------------------------------------------------
# Encoding  ([P1] capability matrix "NF4 pack/unpack + block absmax scales";
#            [P3] QuantizedTensor.data / .scales; readings R2-R5)
# ---------------------------------------------------------------------------

def nearest_code(v: np.ndarray) -> np.ndarray:
    """Index of the nearest NF4 level to each fp32 value, lower index on ties.

    Brute force over all sixteen levels.  Distances are taken in fp64: for
    any v within reach of a decision midpoint (|v| >= 0.03) both v and the
    levels are fp32 numbers within a factor 2^6 of each other, so each
    difference is exact in fp64 and an exact tie compares equal; np.argmin
    then returns the first (lowest) index, which is the tie rule of R4.
    """
    levels = nf4_levels().astype(np.float64)
    v = np.asarray(v, dtype=np.float32)
    flat = v.reshape(-1)
    out = np.empty(flat.size, dtype=np.uint8)
    step = 1 << 20                      # elementwise; the loop only bounds memory use
    for lo in range(0, flat.size, step):
        chunk = flat[lo:lo + step].astype(np.float64)
        dist = np.abs(chunk[:, None] - levels)
        out[lo:lo + step] = np.argmin(dist, axis=-1)
    return out.reshape(v.shape)


def pack_codes(codes: np.ndarray) -> np.ndarray:
    """Two 4-bit codes per byte, the even element in the high nibble (R5); an
    odd count ends with a byte whose low nibble is 7 (R19)."""
    codes = np.asarray(codes, dtype=np.uint8).reshape(-1)
    if codes.size % 2:
        codes = np.concatenate([codes, np.array([7], dtype=np.uint8)])
    return ((codes[0::2] << 4) | codes[1::2]).astype(np.uint8)


def unpack_codes(packed: np.ndarray) -> np.ndarray:
    packed = np.asarray(packed, dtype=np.uint8).reshape(-1)
    out = np.empty(packed.size * 2, dtype=np.uint8)
    out[0::2] = packed >> 4
    out[1::2] = packed & 0x0F
    return out


def double_quant(absmax: np.ndarray, g=None):
    """Simplified double quant of the block scales (reading R6).

    [P1] "Double quantization (simplified)": the block scales become u8 codes
    with one scale-of-scales; [P3] stores them as scales_quantized (u8) and
    scales_scales (f32).  The scale of scales belongs to the whole tensor:
    `g`, when given, is the max over all of the tensor's block scales (for a
    part of a tensor whose other blocks are elsewhere); by default it is the
    max of `absmax` itself.
    """
    absmax = np.asarray(absmax, dtype=np.float32)
    if g is None:
        g = np.float32(absmax.max()) if absmax.size else np.float32(0.0)
    g = np.float32(g)
    if g == 0.0:
        return np.zeros(absmax.size, dtype=np.uint8), np.float32(0.0)
    s_g = np.float32(g / np.float32(255.0))
    ratio = (absmax / s_g).astype(np.float32)           # IEEE fp32 division
    q = np.clip(np.rint(ratio), 0, 255).astype(np.uint8)  # rint: half to even
    return q, s_g


def quantize(w: np.ndarray, block_size: int = 64, double: bool = False) -> dict:
    """Blockwise NF4 quantization of an fp32 tensor ([P1] quantize_nf4(&w, 64)).

    Returns a dict mirroring the QuantizedTensor fields of [P3]:
    codes (packed u8), absmax (fp32 per block), and with double quant also
    absmax_q (u8 per block) and absmax_scale (fp32).
    """
    w = np.asarray(w, dtype=np.float32)
    flat = w.reshape(-1)
    if block_size <= 0 or block_size % 2:
        raise ValueError("block_size must be a positive even number")
    if not np.all(np.isfinite(flat)):
        raise ValueError("non-finite input")
    # R19: a short last block; zero padding changes neither its absmax nor the
    # codes of its elements, and the padding's own codes are dropped below.
    n = flat.size
    pad = (-n) % block_size
    blocks = np.concatenate([flat, np.zeros(pad, dtype=np.float32)]).reshape(-1, block_size)
    absmax = np.abs(blocks).max(axis=1).astype(np.float32)
    codes = np.full(blocks.shape, 7, dtype=np.uint8)       # R3: absmax == 0
    nz = absmax > 0
    if np.any(nz):
        v = (blocks[nz] / absmax[nz][:, None]).astype(np.float32)  # R4
        codes[nz] = nearest_code(v)
    out = {
        "codes": pack_codes(codes.reshape(-1)[:n]),
        "absmax": absmax,
        "shape": tuple(w.shape),
        "block_size": int(block_size),
    }
    if double:
        q, s_g = double_quant(absmax)
        out["absmax_q"] = q
        out["absmax_scale"] = np.float32(s_g)
    return out


def block_scales(q: dict, use_double: bool | None = None) -> np.ndarray:
    """The fp32 scale each block is decoded with (absmax, or q * s_g)."""
    if use_double is None:
        use_double = "absmax_q" in q
    if use_double:
        return (q["absmax_q"].astype(np.float32) * np.float32(q["absmax_scale"])).astype(np.float32)
    return np.asarray(q["absmax"], dtype=np.float32)


# ---------------------------------------------------------------------------
# Dequantization  ([P1] "Honor compute_dtype (BF16/F16/F32) in forward
#                  dequant"; dequantize_nf4; reading R7)
# ---------------------------------------------------------------------------

def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even); returns the uint16 bits.

    Written on the uint32 view: add 0x7FFF plus the lowest kept bit, then drop
    the low 16 bits.  NaN is kept quiet.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    rounded = ((u + 0x7FFF + lsb) >> 16).astype(np.uint32)
    nan = np.isnan(x)
    rounded = np.where(nan, ((u >> 16) | 0x40).astype(np.uint32), rounded)
    return rounded.astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    bits = np.asarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32)


def dequantize(q: dict, out_dtype: str = "f32") -> np.ndarray:
    """w' = fp32(L[code] * scale) per element, reshaped to the stored shape.

    out_dtype "f32" gives fp32, "bf16" gives the uint16 bit patterns of the
    RNE-rounded values, "f16" gives numpy float16 (RNE).
    """
    levels = nf4_levels()
    n = int(np.prod(q["shape"]))
    codes = unpack_codes(q["codes"])[:n]
    scales = block_scales(q)
    bs = q["block_size"]
    per_elem_scale = np.repeat(scales, bs)[:n]
    w = (levels[codes] * per_elem_scale).astype(np.float32)   # one fp32 product
    w = w.reshape(q["shape"])
    if out_dtype == "f32":
        return w
    if out_dtype == "bf16":
        return bf16_round(w).reshape(q["shape"])
    if out_dtype == "f16":
        with np.errstate(over="ignore"):   # beyond the f16 range: +-inf, as IEEE rounding gives
            return w.astype(np.float16)
    raise ValueError(out_dtype)


# ---------------------------------------------------------------------------
# QLoRA linear  ([P4] equation 6.3.6 and "Rank, alpha, and target modules";
#                [P2] scale() = alpha / r; [P1] QuantizedLinear::forward;
#                readings R8, R9)
# ---------------------------------------------------------------------------

def qlora_forward(x, w_hat, a, b, alpha: float, bias=None):
    """y = x W'^T + (alpha/r) (x A^T) B^T (+ bias), all in fp64.

    x [M, K], w_hat [N, K] (the bf16-rounded dequantized base, as floats),
    a [r, K], b [N, r].  Returns (y, t) with t = x A^T unscaled.
    """
    x = np.asarray(x, dtype=np.float64)
    w_hat = np.asarray(w_hat, dtype=np.float64)
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    r = a.shape[0]
    s = float(alpha) / float(r)
    t = x @ a.T
    y = x @ w_hat.T + s * (t @ b.T)
    if bias is not None:
        y = y + np.asarray(bias, dtype=np.float64)[None, :]
    return y, t


def qlora_backward(x, w_hat, a, b, alpha: float, dy):
    """Adapter gradients and input gradient for L = sum(dy * y), W frozen.

    Returns (dA [r, K], dB [N, r], dx [M, K]) in fp64:
      t = x A^T, u = dy B,
      dB = s dy^T t,  dA = s u^T x,  dx = dy W' + s u A.
    """
    x = np.asarray(x, dtype=np.float64)
    w_hat = np.asarray(w_hat, dtype=np.float64)
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    dy = np.asarray(dy, dtype=np.float64)
    r = a.shape[0]
    s = float(alpha) / float(r)
    t = x @ a.T
    u = dy @ b
    d_b = s * (dy.T @ t)
    d_a = s * (u.T @ x)
    d_x = dy @ w_hat + s * (u @ a)
    return d_a, d_b, d_x


# ---------------------------------------------------------------------------
# Merge  ([P3] merge_and_export_gguf: W_merged = W_base + (B @ A) * scale;
#         [P4] "The merge math", equation 6.3.6; reading R16)
# ---------------------------------------------------------------------------

def merge(q: dict, a, b, alpha: float, out_dtype: str = "bf16") -> np.ndarray:
    """Dense merged weight W' + (alpha/r) B A of a quantized base.

    W' is the fp32 dequant; B A and the sum are exact in fp64.  out_dtype
    "f64" returns that sum, "f32" its round to fp32, "bf16" the uint16 bits of
    the fp32 value rounded to bf16, "f16" the fp32 value rounded to f16 (R16;
    the f16 output is the pages' F16 compute dtype applied to the merge).
    """
    w = dequantize(q, "f32").astype(np.float64)
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    s = float(alpha) / float(a.shape[0])
    merged = w + s * (b @ a)
    if out_dtype == "f64":
        return merged
    m32 = merged.astype(np.float32)
    if out_dtype == "f32":
        return m32
    if out_dtype == "bf16":
        return bf16_round(m32).reshape(merged.shape)
    if out_dtype == "f16":
        with np.errstate(over="ignore"):   # beyond the f16 range: +-inf, as IEEE rounding gives
            return m32.astype(np.float16)
    raise ValueError(out_dtype)


def matmul_bruteforce(p, q):
    """Plain triple loop p @ q in Python floats (for tiny pinning cases)."""
    p = np.asarray(p, dtype=np.float64)
    q = np.asarray(q, dtype=np.float64)
    n, k = p.shape
    k2, m = q.shape
    assert k == k2
    out = np.zeros((n, m), dtype=np.float64)
    pl = p.tolist()
    ql = q.T.tolist()
    for i in range(n):
        row = pl[i]
        for j in range(m):
            col = ql[j]
            acc = 0.0
            for kk in range(k):
                acc += row[kk] * col[kk]
            out[i, j] = acc
    return out
