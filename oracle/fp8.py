"""FP8 (e4m3fn) per-tensor quantisation, fp64 emulation — test infrastructure.

[AP-lin]: with --fp8 "most layers" become Float8Linear with per-tensor
scaling.  The pages give nothing more; the reading used here is dynamic
scaling from the tensor's own absolute maximum, s = 448 / amax, values
rounded to the nearest e4m3fn value (ties to even) and saturated at ±448.

e4m3fn: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits, no
infinities; largest finite 448; smallest normal 2^-6; subnormal spacing 2^-9.

bfloat16 (the activation dtype of the bf16 and FP8 configurations, [AP-lin]):
1 sign bit, 8 exponent bits (bias 127), 7 stored mantissa bits; largest finite
(2 - 2^-7) * 2^127; smallest normal 2^-126; subnormal spacing 2^-133.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
_MIN_NORMAL_EXP = -6   # smallest normal is 2^-6
_MANT_BITS = 3


def e4m3_round(x: np.ndarray) -> np.ndarray:
    """Nearest e4m3fn value to each element (ties to even), saturating to ±448."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    # binade exponent e with 2^e <= a < 2^(e+1); below the normal range the
    # spacing stays that of the smallest binade (subnormals)
    _, ex = np.frexp(np.maximum(a, 2.0 ** _MIN_NORMAL_EXP))
    e = ex.astype(np.float64) - 1.0
    ulp = np.exp2(e - _MANT_BITS)
    y = np.round(a / ulp) * ulp          # numpy rounds halves to even
    y = np.minimum(y, E4M3_MAX)
    return np.copysign(y, x)


BF16_MAX = (2.0 - 2.0 ** -7) * 2.0 ** 127


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Nearest bfloat16 value to each element (ties to even); beyond the
    largest finite value the result is +-inf (round-to-nearest overflow)."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    _, ex = np.frexp(np.maximum(a, 2.0 ** -126))
    ulp = np.exp2(ex.astype(np.float64) - 1.0 - 7.0)
    y = np.round(a / ulp) * ulp          # numpy rounds halves to even
    y = np.where(y > BF16_MAX, np.inf, y)
    return np.copysign(y, x)


# Where floating point decides an FP8 code, the decision is taken in single
# precision, the precision of the quantising kernel: the tensor's values and
# amax in fp32, the scale qmax / amax as one correctly rounded fp32 division,
# each product value * scale rounded to fp32, and that fp32 value rounded to
# the FP8 format.  (A value exactly on an FP8 midpoint otherwise rounds one way
# in fp32 and the other in fp64.)  Dequantisation and accumulation stay fp64.

def _f32(x):
    return np.asarray(x, dtype=np.float64).astype(np.float32)


def fp8_scale(t: np.ndarray, qmax: float = E4M3_MAX) -> float:
    """Per-tensor scale qmax / max|t| in fp32 (a floor keeps an all-zero tensor finite)."""
    t32 = _f32(t)
    amax = np.float32(np.max(np.abs(t32))) if t32.size else np.float32(0.0)
    return float(np.float32(qmax) / np.maximum(amax, np.float32(1e-12)))


def _scaled(t: np.ndarray, s: float) -> np.ndarray:
    """fp32 products t * s (s an fp32 value), as fp64."""
    return (_f32(t) * np.float32(s)).astype(np.float64)


def quantize_e4m3(t: np.ndarray) -> tuple[np.ndarray, float]:
    """Return (codes as fp64 values, scale) with t ~= codes / scale."""
    s = fp8_scale(t)
    return e4m3_round(_scaled(t, s)), s


def fp8_matmul(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """a @ b with both operands quantised per tensor to e4m3, fp64 accumulate."""
    qa, sa = quantize_e4m3(a)
    qb, sb = quantize_e4m3(b)
    return (qa @ qb) / (sa * sb)


# ------------------------------------------------------------ e5m2 (NEXT-4)
# The gradient variant of the FP8 recipe: e5m2 (1 sign, 5 exponent bits with
# bias 15, 2 mantissa bits; largest finite 57344, smallest normal 2^-14,
# subnormal spacing 2^-16) for the gradient operand of the input-gradient
# GEMMs, the weight operand staying e4m3.  Reading (the pages name FP8 with
# per-tensor scaling only): scale 57344 / amax, round to nearest (ties to
# even), saturate at the largest finite value.

E5M2_MAX = 57344.0


def e5m2_round(x: np.ndarray) -> np.ndarray:
    """Nearest e5m2 value to each element (ties to even), saturating to ±57344."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    _, ex = np.frexp(np.maximum(a, 2.0 ** -14))
    e = ex.astype(np.float64) - 1.0
    ulp = np.exp2(e - 2)
    y = np.minimum(np.round(a / ulp) * ulp, E5M2_MAX)
    return np.copysign(y, x)


def quantize_e5m2(t: np.ndarray) -> tuple[np.ndarray, float]:
    """Return (codes as fp64 values, scale) with t ~= codes / scale, scale = 57344 / amax (fp32)."""
    s = fp8_scale(t, E5M2_MAX)
    return e5m2_round(_scaled(t, s)), s


def fp8_matmul_grad(g: np.ndarray, w: np.ndarray) -> np.ndarray:
    """g @ w with the gradient g quantised per tensor to e5m2 and the weight w to
    e4m3, fp64 accumulate (an input-gradient GEMM of the e5m2 variant)."""
    qg, sg = quantize_e5m2(g)
    qw, sw = quantize_e4m3(w)
    return (qg @ qw) / (sg * sw)


# ------------------------------------------------- fixed-scale quantisation
def quantize_fixed(t: np.ndarray, scale: float, fmt: str = "e4m3") -> np.ndarray:
    """Codes (as fp64 values) of t * scale rounded to e4m3 or e5m2, for a tensor
    whose per-tensor scale is known in advance rather than measured (scale an
    fp32 value; the product is rounded to fp32 first, as above)."""
    r = e4m3_round if fmt == "e4m3" else e5m2_round
    return r(_scaled(t, scale))


def bound_scale(qmax: float, n: int) -> float:
    """The fp32 scale qmax / (1/n) of a tensor bounded by 1/n in magnitude:
    1/n rounded to fp32, then one fp32 division."""
    inv_n = np.float32(1.0) / np.float32(n)
    return float(np.float32(qmax) / inv_n)
