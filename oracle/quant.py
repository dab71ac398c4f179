"""FP8 (e4m3) quantisation of expert weights and activations (oracle side, test infrastructure).

[pl] lists the weight formats the model ships in (BF16, FP8 and NVFP4, with their memory
footprints) and [course] table 2.2 quotes the fp8 speed on one H100; neither page gives the
scheme, so the plainest symmetric one is read here:

  * Element format e4m3 (the "fn" variant): one sign bit, four exponent bits with bias 7 and
    three mantissa bits.  Exponent field 0 holds the subnormals m/8 * 2^-6; the largest finite
    magnitude is 448 (pattern 0x7E); patterns 0x7F and 0xFF are NaN; there is no infinity.
  * Every row v (one output row of an expert weight matrix, or one token's activation row where
    it enters an expert GEMM) has one binary32 scale s = max|v| / 448 (a binary32 division).
    Its codes are the e4m3 values nearest (ties to the even significand) to the binary32
    quotients v / s, clamped to +-448.  An all-zero row has s = 0 and zero codes.
  * An expert GEMM multiplies codes and applies the two scales to the sum:
        y[t, r] = s_w[r] * s_x[t] * sum_k q_w[r, k] q_x[t, k].
  * Activations are quantised where they enter an expert GEMM: the stored (bf16) normed hidden
    state, once per token, and the stored (bf16) SiLU-GLU output h, once per token-slot.

Pinned in tests/test_oracle_quant.py: the 256-code table against the format definition written
independently as bit fields, rounding against torch's float8_e4m3fn conversion on every binary32
neighbourhood of the grid, ties, saturation, the error bound of a row quantisation, and the fp8
MoE against the bf16 MoE when every operand already lies on the e4m3 grid.
"""
import numpy as np

E4M3_MAX = 448.0
_MIN_NORMAL_EXP = -6  # 2^-6 is the smallest normal magnitude


def e4m3_table():
    """The value of each of the 256 codes (float64; NaN for 0x7F and 0xFF)."""
    out = np.empty(256, dtype=np.float64)
    for c in range(256):
        sign = -1.0 if c & 0x80 else 1.0
        e = (c >> 3) & 0xF
        m = c & 0x7
        if e == 0xF and m == 0x7:
            out[c] = np.nan
        elif e == 0:
            out[c] = sign * (m / 8.0) * 2.0 ** _MIN_NORMAL_EXP
        else:
            out[c] = sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return out


def round_e4m3(v):
    """Nearest e4m3 value to each element of v (ties to even significand), clamped to +-448.

    Returns float64 values on the e4m3 grid; the sign of a value that rounds to zero is kept.
    """
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    _, ex = np.frexp(np.maximum(a, 2.0 ** _MIN_NORMAL_EXP))  # a = f * 2^ex, f in [0.5, 1)
    binade = np.minimum(ex - 1, 8)                            # floor(log2 a), subnormals at -6
    quantum = np.ldexp(1.0, binade - 3)                       # grid spacing: 3 mantissa bits
    r = np.rint(a / quantum) * quantum                        # rint: halves go to the even integer
    r = np.minimum(r, E4M3_MAX)
    return np.copysign(r, v)


def encode_e4m3(values):
    """Codes (uint8) of values that lie on the e4m3 grid (as returned by round_e4m3).

    Codes 0x00..0x7E are the non-negative values in increasing order, so a magnitude's code is
    its rank among them; the sign bit is 0x80.  Raises if a value is not on the grid.
    """
    values = np.asarray(values, dtype=np.float64)
    mags = e4m3_table()[:0x7F]
    a = np.abs(values)
    code = np.searchsorted(mags, a).astype(np.int64)
    if np.any(code > 0x7E) or not np.array_equal(mags[np.minimum(code, 0x7E)], a):
        raise ValueError("value not on the e4m3 grid")
    code = code | np.where(np.signbit(values), 0x80, 0)
    return code.astype(np.uint8)


def decode_e4m3(codes):
    """Values (float64) of e4m3 codes."""
    return e4m3_table()[np.asarray(codes, dtype=np.uint8)]


def quantize_rows(v):
    """Per-row e4m3 quantisation of a 2-D array of binary32-representable values.

    Returns (values on the e4m3 grid float64 [n, k], scales float32 [n]); the dequantised row
    is values * scale.  Codes are `encode_e4m3(values)`.
    """
    v = np.ascontiguousarray(np.asarray(v, dtype=np.float64).astype(np.float32))
    if v.ndim != 2:
        raise ValueError("quantize_rows takes a 2-D array")
    amax = np.max(np.abs(v), axis=1) if v.shape[1] else np.zeros(v.shape[0], np.float32)
    scale = (amax / np.float32(E4M3_MAX)).astype(np.float32)  # binary32 division
    q = np.zeros(v.shape, dtype=np.float64)
    nz = scale > 0
    quo = (v[nz] / scale[nz, None]).astype(np.float32)          # binary32 division per element
    q[nz] = round_e4m3(quo.astype(np.float64))
    return q, scale


def quantize_matrix(w):
    """Row-wise quantisation of a weight matrix or a stack of them ([..., rows, k]).

    Returns (values float64 of the same shape, scales float32 [..., rows]).
    """
    w = np.asarray(w)
    lead = w.shape[:-1]
    q, s = quantize_rows(w.reshape(-1, w.shape[-1]))
    return q.reshape(w.shape), s.reshape(lead)
