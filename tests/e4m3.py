"""e4m3 (fp8: 1 sign, 4 exponent bits with bias 7, 3 mantissa bits, no infinities, NaN =
S.1111.111, largest finite 448) written out in numpy for the tests: decoding bytes and
rounding to nearest even with saturation, the rounding the kernels get from cvt.rn.satfinite."""
import numpy as np

E4M3_MAX = 448.0


def decode(b: np.ndarray) -> np.ndarray:
    b = np.asarray(b, dtype=np.uint8).astype(np.int64)
    s = np.where(b & 0x80, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = (b & 7).astype(np.float64)
    val = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    val = np.where((e == 15) & ((b & 7) == 7), np.nan, val)
    return s * val


def quantize(x: np.ndarray) -> np.ndarray:
    """Nearest e4m3 value, ties to even mantissa, |x| clamped to 448."""
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), E4M3_MAX)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -6)))        # binade (subnormals share 2^-6's step)
    step = np.exp2(e - 3.0)
    q = np.rint(a / step) * step                             # np.rint rounds half to even
    q = np.minimum(q, E4M3_MAX)
    return np.sign(x) * q


def random_bytes(rng, shape, max_exp: int = 9) -> np.ndarray:
    """Random finite e4m3 codes with exponent field 1..max_exp (|value| < 2^(max_exp-6))."""
    s = rng.integers(0, 2, size=shape) << 7
    e = rng.integers(1, max_exp + 1, size=shape) << 3
    m = rng.integers(0, 8, size=shape)
    return (s | e | m).astype(np.uint8)


def encode(q: np.ndarray) -> np.ndarray:
    """Bytes of values that are already e4m3 numbers (e.g. quantize's output)."""
    q = np.asarray(q, dtype=np.float64)
    s = (q < 0).astype(np.int64) << 7
    a = np.abs(q)
    sub = a < 2.0 ** -6
    e = np.where(sub, 0, np.floor(np.log2(np.where(sub, 1.0, a))) + 7).astype(np.int64)
    m = np.where(sub, np.rint(a / 2.0 ** -9), np.rint((a / np.exp2(e - 7.0) - 1.0) * 8.0)).astype(np.int64)
    return (s | (e << 3) | m).astype(np.uint8)


def quantize_tensor(x: np.ndarray):
    """Per-tensor scaling as FP8 attention uses it: descale = max|x| / 448, bytes of
    e4m3(x / descale).  Returns (bytes, descale)."""
    amax = float(np.abs(x).max())
    descale = amax / E4M3_MAX if amax > 0 else 1.0
    return encode(quantize(x / descale)), descale
