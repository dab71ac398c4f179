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

Pinned in tests/test_oracle_quant.py: the 256-code table against torch's float8_e4m3fn bit
patterns, rounding against torch's conversion on every binary32 neighbourhood of the grid, ties,
saturation, the error bound of a row quantisation, and the fp8 MoE against the bf16 MoE when every
operand already lies on the e4m3 grid.  The NVFP4 part at the end (e2m1 elements with e4m3 block
scales) is pinned by brute-force nearest rounding, on-grid identity, a closed-form error bound
and the bf16 expert on grid operands.
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


# ---- NVFP4: e2m1 elements with one e4m3 scale per 16-element block ----------------------------
#
# The pages name NVFP4 as the 4-bit weight format (18 GB, [pl]) that Blackwell kernels run
# ([blog], "NVFP4 kernels"), without its arithmetic.  Read here as: elements e2m1 (a sign bit,
# two exponent bits with bias 1, one mantissa bit: 0, 0.5, 1, 1.5, 2, 3, 4, 6); every 16
# consecutive elements of a row along K share one e4m3 block scale; every row has one binary32
# scale g = max|row| / (6 * 448), so that the block scales use the e4m3 range.  With a = max|block|:
#     s_b  = e4m3(a / 6 / g)                  (binary32 divisions, RNE to e4m3, clamped)
#     code = e2m1(x / (s_b * g))              (binary32 product and division, RNE, clamped to 6)
# and the dequantised element is code * s_b * g.  A block whose scale rounds to 0 has zero codes.

E2M1_MAX = 6.0
NVFP4_BLOCK = 16


def e2m1_table():
    """The value of each of the 16 e2m1 codes (bit 3 sign, bits 2-1 exponent, bit 0 mantissa)."""
    out = np.empty(16, dtype=np.float64)
    for c in range(16):
        sign = -1.0 if c & 0x8 else 1.0
        e = (c >> 1) & 0x3
        m = c & 0x1
        out[c] = sign * (m * 0.5 if e == 0 else (1.0 + m / 2.0) * 2.0 ** (e - 1))
    return out


def round_e2m1(v):
    """Nearest e2m1 value (ties to the even mantissa), clamped to +-6; float64 out."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    _, ex = np.frexp(np.maximum(a, 1.0))        # binades [1,2), [2,4), [4,8); below 1 as [1,2)
    binade = np.minimum(ex - 1, 2)
    quantum = np.ldexp(1.0, binade - 1)         # one mantissa bit: spacing 0.5, 1, 2
    r = np.minimum(np.rint(a / quantum) * quantum, E2M1_MAX)
    return np.copysign(r, v)


def encode_e2m1(values):
    """Codes (uint8, 0..15) of values on the e2m1 grid."""
    values = np.asarray(values, dtype=np.float64)
    mags = e2m1_table()[:8]
    a = np.abs(values)
    code = np.searchsorted(mags, a).astype(np.int64)
    if np.any(code > 7) or not np.array_equal(mags[np.minimum(code, 7)], a):
        raise ValueError("value not on the e2m1 grid")
    return (code | np.where(np.signbit(values), 0x8, 0)).astype(np.uint8)


def quantize_nvfp4_rows(v):
    """NVFP4 quantisation of a 2-D array of binary32-representable values, k % 16 == 0.

    Returns (element values on the e2m1 grid float64 [n, k], block scales on the e4m3 grid
    float64 [n, k / 16], row scales float32 [n]); the dequantised row is
    values * repeat(block scales, 16) * row scale.
    """
    v = np.ascontiguousarray(np.asarray(v, dtype=np.float64).astype(np.float32))
    n, k = v.shape
    if k % NVFP4_BLOCK:
        raise ValueError("row length must be a multiple of 16")
    amax = np.max(np.abs(v), axis=1) if k else np.zeros(n, np.float32)
    g = (amax / np.float32(E2M1_MAX * E4M3_MAX)).astype(np.float32)
    blocks = v.reshape(n, k // NVFP4_BLOCK, NVFP4_BLOCK)
    bmax = np.max(np.abs(blocks), axis=2)
    sb = np.zeros(bmax.shape, dtype=np.float64)
    q = np.zeros(blocks.shape, dtype=np.float64)
    rows = g > 0
    t = (bmax[rows] / np.float32(E2M1_MAX)).astype(np.float32)
    t = (t / g[rows, None]).astype(np.float32)
    sb[rows] = round_e4m3(t.astype(np.float64))
    step = (sb.astype(np.float32) * g[:, None]).astype(np.float32)   # binary32 product
    live = step > 0
    quo = (blocks[live] / step[live][:, None]).astype(np.float32)
    q[live] = round_e2m1(quo.astype(np.float64))
    return q.reshape(n, k), sb, g


def dequantize_nvfp4(q, sb, g):
    """code * block scale * row scale (float64)."""
    q = np.asarray(q, dtype=np.float64)
    n, k = q.shape
    s = np.repeat(np.asarray(sb, dtype=np.float64), NVFP4_BLOCK, axis=1)
    return q * s * np.asarray(g, dtype=np.float64)[:, None]
