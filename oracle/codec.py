"""ctypes front end of the C oracle codec (``nf4_oracle.c``).

TEST INFRASTRUCTURE ONLY (see the package docstring).

Pages followed:
  "LoRA 与 QLoRA" (whoami-wesleyyou.top), QLoRA sections "1. NF4" and
  "2. Double Quantization (DQ)";
  "QLoRA: Efficient Finetuning of Quantized LLMs" deck "3 QLoRA Finetuning"
  (learn.ifs.name), cards 1-4;
  jjjymmm.cn 2024/03 QLoRA post, sections "4-bit NormalFloat(NF4)",
  "Double Quantization" and "QLoRA".
"""
import ctypes

import numpy as np

from . import build as _build

#: Offset of the outermost quantile.  The pages do not print it; the printed
#: NF4 table (jjjymmm.cn, "4-bit NormalFloat(NF4)") pins it to [0.96768,
#: 0.96773].  This closed form, halfway between the half-bin offsets of 16 and
#: 15 equal-mass bins, lies in that window.
DELTA = 1.0 - 0.5 * (1.0 / 32.0 + 1.0 / 30.0)

BLOCK = 64        # weights per absmax block ("LoRA 与 QLoRA", DQ: 64 weights)
DQ_GROUP = 256    # block constants per DQ scale (deck card 4; jjjymmm.cn DQ)

_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(_build.build())
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        L.oracle_normal_cdf.restype = ctypes.c_double
        L.oracle_normal_cdf.argtypes = [ctypes.c_double]
        L.oracle_normal_quantile.restype = ctypes.c_double
        L.oracle_normal_quantile.argtypes = [ctypes.c_double]
        L.oracle_nf4_codebook.restype = None
        L.oracle_nf4_codebook.argtypes = [ctypes.c_double, P, P]
        L.oracle_nf4_nearest.restype = ctypes.c_int
        L.oracle_nf4_nearest.argtypes = [ctypes.c_float, P]
        L.oracle_nf4_quantize.restype = None
        L.oracle_nf4_quantize.argtypes = [P, I64, P, P, P]
        L.oracle_nf4_double_quant.restype = None
        L.oracle_nf4_double_quant.argtypes = [P, I64, ctypes.c_float, P, P]
        L.oracle_dq_restore.restype = ctypes.c_float
        L.oracle_dq_restore.argtypes = [ctypes.c_int8, ctypes.c_float, ctypes.c_float]
        L.oracle_bf16_rn.restype = ctypes.c_uint16
        L.oracle_bf16_rn.argtypes = [ctypes.c_float]
        L.oracle_nf4_dequant.restype = None
        L.oracle_nf4_dequant.argtypes = [P, I64, P, P, P, P, P, P]
        L.oracle_nf4_dequant_f32.restype = None
        L.oracle_nf4_dequant_f32.argtypes = [P, I64, P, P, P, P, P, P]
        L.oracle_e4m3_value.restype = ctypes.c_double
        L.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_encode.restype = ctypes.c_uint8
        L.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        L.oracle_nf4_double_quant_e4m3.restype = None
        L.oracle_nf4_double_quant_e4m3.argtypes = [P, I64, ctypes.c_float, P, P]
        L.oracle_dq_restore_e4m3.restype = ctypes.c_float
        L.oracle_dq_restore_e4m3.argtypes = [ctypes.c_uint8, ctypes.c_float, ctypes.c_float]
        L.oracle_nf4_dequant_fmt.restype = None
        L.oracle_nf4_dequant_fmt.argtypes = [P, I64, P, P, ctypes.c_int, P, P, P, P]
        L.oracle_nf4_dequant_f32_fmt.restype = None
        L.oracle_nf4_dequant_f32_fmt.argtypes = [P, I64, P, P, ctypes.c_int, P, P, P, P]
        _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def normal_quantile(p: float) -> float:
    """Q_Z(p) of N(0,1) by bisection ("LoRA 与 QLoRA", Gaussian 假设与分位数)."""
    return lib().oracle_normal_quantile(float(p))


def normal_cdf(x: float) -> float:
    return lib().oracle_normal_cdf(float(x))


def codebook(delta: float = DELTA):
    """The 16 NF4 values, ascending: (float64 array, float32 array).

    Asymmetric halves sharing one zero (deck card 3), normalized by the largest
    quantile so the ends are exactly +-1 ("LoRA 与 QLoRA", 归一化与匹配)."""
    c64 = np.zeros(16, np.float64)
    c32 = np.zeros(16, np.float32)
    lib().oracle_nf4_codebook(float(delta), _ptr(c64), _ptr(c32))
    return c64, c32


_CB32 = None


def cb32():
    global _CB32
    if _CB32 is None:
        _CB32 = codebook()[1]
    return _CB32


def nearest(x: float, cb=None) -> int:
    cb = cb32() if cb is None else _c(cb, np.float32)
    return lib().oracle_nf4_nearest(ctypes.c_float(x), _ptr(cb))


def quantize(w):
    """fp32 weights (any shape and numel >= 1, flattened row-major) ->
    (codes uint8 [ceil(numel/2)], absmax fp32 [ceil(numel/64)]).

    jjjymmm.cn "4-bit NormalFloat(NF4)": divide by the block ABSMAX, take the
    nearest quant-book value; "LoRA 与 QLoRA" DQ: one constant per 64 weights.
    A last, partial block takes its absmax over the weights it has; an odd
    numel leaves code 7 (a zero weight's code) in the last low nibble."""
    w = _c(w, np.float32).reshape(-1)
    n = w.size
    if n < 1:
        raise ValueError("numel must be positive")
    codes = np.zeros((n + 1) // 2, np.uint8)
    absmax = np.zeros((n + BLOCK - 1) // BLOCK, np.float32)
    cb = cb32()
    lib().oracle_nf4_quantize(_ptr(w), n, _ptr(cb), _ptr(codes), _ptr(absmax))
    return codes, absmax


def widen16(bits, kind: str):
    """16-bit weights (bit patterns, uint16) -> their exact fp32 values.

    The pages warn against loading a 16-bit checkpoint and then quantizing it
    carelessly ("LoRA 与 QLoRA", QLoRA usage notes); the method itself is
    defined on real weights, and every bf16 or fp16 value is exactly a binary32
    value, so a 16-bit weight enters the quantizer as that value.
      kind "bf16": the 16 bits are the top half of the binary32 pattern;
      kind "f16":  IEEE binary16 -> binary32 (exact, subnormals included)."""
    b = np.ascontiguousarray(bits, np.uint16).reshape(-1)
    if kind == "bf16":
        return (b.astype(np.uint32) << 16).view(np.float32)
    if kind == "f16":
        return _f16_to_f32(b)
    raise ValueError(kind)


def _f16_to_f32(b):
    """binary16 bits -> binary32, written out from the two formats' fields."""
    b = b.astype(np.uint32)
    sign = (b >> 15) << 31
    exp = (b >> 10) & 0x1F
    man = b & 0x3FF
    out = np.zeros(b.size, np.uint32)
    normal = (exp > 0) & (exp < 31)
    out[normal] = sign[normal] | ((exp[normal] + (127 - 15)) << 23) | (man[normal] << 13)
    special = exp == 31  # inf / NaN keep their payload
    out[special] = sign[special] | (0xFF << 23) | (man[special] << 13)
    zero = (exp == 0) & (man == 0)
    out[zero] = sign[zero]
    sub = (exp == 0) & (man != 0)  # value man * 2^-24: normalise
    for i in np.nonzero(sub)[0]:
        m, e = int(man[i]), -14
        while not (m & 0x400):
            m <<= 1
            e -= 1
        out[i] = int(sign[i]) | ((e + 127) << 23) | ((m & 0x3FF) << 13)
    return out.view(np.float32)


def quantize16(bits, kind: str):
    """quantize() of 16-bit weights: the exact fp32 values (widen16), quantized."""
    return quantize(widen16(bits, kind))


def exact_sum_units(a) -> int:
    """The exact sum of binary32 values, as an integer count of 2^-149.

    Every finite binary32 value is m * 2^(s - 149) with an integer m < 2^24
    and s = max(exponent field, 1) - 1 (subnormals have s = 0), so the sum is
    the integer sum of m * 2^s: summed exactly per exponent (numpy int64, at
    most 2^24 per term), then shifted into one Python integer."""
    bits = _c(a, np.float32).reshape(-1).view(np.uint32)
    e = ((bits >> 23) & 0xFF).astype(np.int64)
    f = (bits & 0x7FFFFF).astype(np.int64)
    m = np.where(e > 0, f | 0x800000, f)
    m = np.where((bits >> 31) == 1, -m, m)
    s = np.maximum(e, 1) - 1
    total = 0
    for sv in np.unique(s):
        total += int(m[s == sv].sum(dtype=np.int64)) << int(sv)
    return total


def nearest_f32(num: int, den: int) -> np.float32:
    """The binary32 value nearest to (num / den) * 2^-149, ties to even.

    Binary32 values below 2^-125 are the integers 0 .. 2^24 in units of
    2^-149 and their bit pattern is that integer; above, a value with leading
    bit p (p >= 24) keeps 24 significant bits, a quantum of 2^(p - 23) units,
    and has exponent field p - 22 (a significand that rounds up to 2^24 carries
    into the exponent through the same formula)."""
    if den <= 0:
        raise ValueError("den must be positive")
    neg = num < 0
    num = -num if neg else num
    p = num // den
    p = p.bit_length() - 1 if p > 0 else -1   # leading bit of floor(num / den)
    shift = max(0, p - 23)
    d = den << shift                          # quantum of 2^shift units
    k, rem = divmod(num, d)
    if 2 * rem > d or (2 * rem == d and (k & 1)):
        k += 1
    bits = k if shift == 0 else ((shift + 1) << 23) + (k - (1 << 23))
    if bits >= 0x7F800000:
        bits = 0x7F800000                     # beyond the largest finite value
    return np.array([bits | (0x80000000 if neg else 0)], np.uint32).view(np.float32)[0]


def dq_mean(absmax) -> np.float32:
    """mu of the double quantization: the mean of the block constants
    ("LoRA 与 QLoRA", section 2, DQ: subtract the mean mu; mu kept in 32 bits),
    read as the binary32 value nearest to the exact mean, ties to even."""
    a = _c(absmax, np.float32).reshape(-1)
    if a.size < 1:
        raise ValueError("no block constants")
    return nearest_f32(exact_sum_units(a), a.size)


def double_quant(absmax, fmt: str = "int8"):
    """fp32 block constants -> (qabs [nb], scale fp32 [ceil(nb/256)], mu fp32).

    "LoRA 与 QLoRA" DQ: r_j = (a_j - mu)/b, 8-bit rhat_j, mu and b in 32 bits;
    deck card 4 / jjjymmm.cn DQ: blocks of 256 constants.
    fmt "int8": rhat = clamp(rint(r), -127, 127), b = max|d| / 127 (int8 array);
    fmt "e4m3": deck card 4's "8-bit floats": rhat = E4M3(r) (nearest-even,
    saturating), b = max|d| / 448 (uint8 array of E4M3 codes)."""
    a = _c(absmax, np.float32).reshape(-1)
    nb = a.size
    ng = (nb + DQ_GROUP - 1) // DQ_GROUP
    scale = np.zeros(ng, np.float32)
    mu = dq_mean(a)
    if fmt == "int8":
        qabs = np.zeros(nb, np.int8)
        lib().oracle_nf4_double_quant(_ptr(a), nb, ctypes.c_float(mu), _ptr(qabs), _ptr(scale))
    elif fmt == "e4m3":
        qabs = np.zeros(nb, np.uint8)
        lib().oracle_nf4_double_quant_e4m3(_ptr(a), nb, ctypes.c_float(mu), _ptr(qabs), _ptr(scale))
    else:
        raise ValueError(fmt)
    return qabs, scale, mu


def e4m3_value(code: int) -> float:
    """The value of an OCP FP8 E4M3 code (NaN for 0x7F / 0xFF)."""
    return lib().oracle_e4m3_value(int(code) & 0xFF)


def e4m3_encode(x: float) -> int:
    """binary32 -> E4M3 code: nearest, ties to even mantissa, saturating at +-448."""
    return int(lib().oracle_e4m3_encode(ctypes.c_float(x)))


def dq_restore(qabs, scale, mu, fmt: str = "int8"):
    """ahat_j = fp32(mu + fp32(b_g * rhat_j)) for every j (vector form)."""
    scale = _c(scale, np.float32).reshape(-1)
    L = lib()
    if fmt == "e4m3":
        q = _c(qabs, np.uint8).reshape(-1)
        f = lambda j: L.oracle_dq_restore_e4m3(int(q[j]), float(scale[j // DQ_GROUP]), float(mu))
    else:
        q = _c(qabs, np.int8).reshape(-1)
        f = lambda j: L.oracle_dq_restore(int(q[j]), float(scale[j // DQ_GROUP]), float(mu))
    out = np.empty(q.size, np.float32)
    for j in range(q.size):
        out[j] = f(j)
    return out


def bf16_rn(x: float) -> int:
    return lib().oracle_bf16_rn(ctypes.c_float(x))


def dequant(codes, numel, absmax=None, qabs=None, scale=None, mu=None, fmt: str = "int8"):
    """doubleDequant to BF16 bits (uint16 [numel]).

    jjjymmm.cn "QLoRA": restore the constant first, then the weight with it;
    deck card 1: weights are dequantized to BFloat16 for every matmul.
    Pass ``absmax`` for plain NF4, or ``qabs, scale, mu`` (and the DQ format)
    for NF4 + DQ."""
    codes = _c(codes, np.uint8).reshape(-1)
    out = np.empty(numel, np.uint16)
    mu_arr = None if mu is None else np.array([mu], np.float32)
    q = None if qabs is None else np.ascontiguousarray(qabs).view(np.uint8).reshape(-1)
    lib().oracle_nf4_dequant_fmt(
        _ptr(codes), numel,
        _ptr(None if absmax is None else _c(absmax, np.float32)),
        _ptr(q), 1 if fmt == "e4m3" else 0,
        _ptr(None if scale is None else _c(scale, np.float32)),
        _ptr(mu_arr), _ptr(cb32()), _ptr(out))
    return out


def dequant_f32(codes, numel, absmax=None, qabs=None, scale=None, mu=None, fmt: str = "int8"):
    """As :func:`dequant`, returning the fp32 product before BF16 rounding."""
    codes = _c(codes, np.uint8).reshape(-1)
    out = np.empty(numel, np.float32)
    mu_arr = None if mu is None else np.array([mu], np.float32)
    q = None if qabs is None else np.ascontiguousarray(qabs).view(np.uint8).reshape(-1)
    lib().oracle_nf4_dequant_f32_fmt(
        _ptr(codes), numel,
        _ptr(None if absmax is None else _c(absmax, np.float32)),
        _ptr(q), 1 if fmt == "e4m3" else 0,
        _ptr(None if scale is None else _c(scale, np.float32)),
        _ptr(mu_arr), _ptr(cb32()), _ptr(out))
    return out


def bf16_bits_to_f64(bits):
    """Widen BF16 bit patterns (uint16) exactly to float64."""
    b = np.ascontiguousarray(bits, np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def unpack_codes(codes, numel):
    """uint8 [ceil(numel/2)] -> uint8 [numel] of 4-bit codes (element 2i = high nibble)."""
    c = np.ascontiguousarray(codes, np.uint8).reshape(-1)
    out = np.empty(numel, np.uint8)
    out[0::2] = (c >> 4)[:(numel + 1) // 2]
    out[1::2] = (c & 15)[:numel // 2]
    return out


def constant_bytes(numel: int) -> int:
    """Bytes of quantization constants with DQ: nb int8 codes, one fp32 scale per
    256 constants, one fp32 mean."""
    nb = numel // BLOCK
    ng = (nb + DQ_GROUP - 1) // DQ_GROUP
    return nb * 1 + ng * 4 + 4
