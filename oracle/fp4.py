"""FP4 block quantization: MXFP4 and NVFP4 (oracle side).

Test infrastructure only (see ``oracle/__init__.py``).

Sources: SII release on Metis, feature list (MXFP4 / NVFP4 formats) and
section 2.3 with Fig. 3 (block-wise quantization: every block shares one scale,
and that scale is set by the block's largest magnitude).  The pages give no
bit-level definition; the readings (R11-R13) take the formats from the OCP
Microscaling v1.0 specification (E2M1 elements, E8M0 block scale, 32 elements
per block) and the two-level NVFP4 scheme (E2M1 elements, E4M3 block scale per
16 elements, one float32 tensor scale), with the op order fixed below.

All quantizer arithmetic is IEEE float32 (numpy float32 ops round to nearest
even), in exactly this order, so that GPU kernels fed the same float32 input
produce identical bytes:

MXFP4, per block of 32 along the block axis
    a    = max |x|
    a==0 : scale code 0, element codes 0
    e    = floor(log2 a)            (exact, from the float's exponent)
    se   = clamp(e - 2, -127, 127)  (2 = exponent of 6, the largest E2M1 value)
    code = se + 127                 (E8M0: value 2**(code-127))
    q    = x * 2**-se               (exact)  ->  element = E2M1(q)

NVFP4, per block of 16, with alpha = max |x| over the whole tensor
    s_t  = alpha / 2688  (2688 = 6 * 448; s_t = 1 when alpha == 0)
    t    = (a / s_t) / 6
    d    = E4M3(t)  round to nearest even, saturating at 448
    d==0 : element codes 0
    enc  = 1 / (d * s_t)
    q    = x * enc  ->  element = E2M1(q)

E2M1(q): |q| goes to the nearest of {0, 0.5, 1, 1.5, 2, 3, 4, 6}; a value
exactly half-way goes to the even code; anything above 6 goes to 6; the sign
bit is the sign bit of q (so negative values that round to zero give 0x8).
Codes are 4 bits s|e1 e0|m.  Two codes share a byte: element 2j in the low
nibble, element 2j+1 in the high nibble, along the block axis.

Dequantization: MXFP4 e2m1(code) * 2**se;  NVFP4 e2m1(code) * d * s_t.

Storage ("outer x inner", blocks along inner): for ``axis=1`` a rows x cols
matrix gives outer=rows, inner=cols; for ``axis=0`` outer=cols, inner=rows
(the matrix is quantized as its transpose).  Scales come in two layouts:
linear [outer][inner/bs] and the tensor-core layout used by the block-scaled
MMA, where 128 rows x 4 scale columns form one 512-byte chunk in which row r,
column c sits at byte (r % 32) * 16 + ((r % 128) // 32) * 4 + (c % 4); chunks
are ordered with the scale-column chunk index fastest, then the 128-row group.
The tensor-core layout pads outer to a multiple of 128 and the scale columns to
a whole 256-element K tile (16 scale columns for NVFP4, 8 for MXFP4) with zeros.
"""

import numpy as np

E2M1_MAGNITUDES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
MX_BLOCK = 32
NV_BLOCK = 16
NV_TENSOR_DIV = np.float32(6.0 * 448.0)   # 2688
KTILE = 256                                # elements of K per tensor-core K tile

F32 = np.float32


# --------------------------------------------------------------------------
# element and scale codecs
# --------------------------------------------------------------------------

def e2m1_encode(q):
    """float32 array -> uint8 E2M1 codes (0..15), round to nearest, ties to the
    even code, saturating at 6.  Written from the value set: a magnitude moves
    to code c when it lies above the midpoint between the values of codes c-1
    and c, or exactly on it when c is even."""
    q = np.asarray(q, dtype=F32)
    a = np.abs(q).astype(np.float64)
    code = np.zeros(q.shape, dtype=np.uint8)
    for c in range(1, 8):
        mid = 0.5 * (E2M1_MAGNITUDES[c - 1] + E2M1_MAGNITUDES[c])
        up = (a > mid) | ((a == mid) & (c % 2 == 0))
        code = np.where(up, np.uint8(c), code)
    return code | (np.signbit(q).astype(np.uint8) << 3)


def e2m1_decode(code):
    """uint8 E2M1 codes -> float64 values."""
    code = np.asarray(code, dtype=np.uint8)
    mag = E2M1_MAGNITUDES[code & 7]
    return np.where(code & 8, -mag, mag)


def e4m3_encode(t):
    """Non-negative float values -> E4M3 (OCP FP8 E4M3FN) codes, round to
    nearest even, saturating at 448.  Exponent bias 7, 3 mantissa bits;
    subnormals m * 2**-9."""
    t = np.asarray(t, dtype=np.float64)
    if np.any(t < 0) or np.any(~np.isfinite(t)):
        raise ValueError("E4M3 scale input must be finite and non-negative")
    _, e2 = np.frexp(t)
    e = np.maximum(e2.astype(np.int64) - 1, -6)       # below 2**-6: quantum 2**-9
    quantum = np.ldexp(1.0, e - 3)
    v = np.round(t / quantum) * quantum                # half to even; exact scaling
    v = np.minimum(v, 448.0)                           # satfinite
    code = np.zeros(t.shape, dtype=np.uint8)
    sub = v < 2.0 ** -6
    code = np.where(sub, (v / 2.0 ** -9).astype(np.int64), code)
    _, ve2 = np.frexp(np.where(sub, 1.0, v))
    E = ve2.astype(np.int64) - 1
    mant = np.where(sub, 1.0, v) / np.ldexp(1.0, E)    # in [1, 2)
    m3 = np.round((mant - 1.0) * 8.0).astype(np.int64)
    normal = ((E + 7) << 3) | m3
    code = np.where(sub, code, normal)
    return code.astype(np.uint8)


def e4m3_decode(code):
    """E4M3 codes (unsigned use, 0x00..0x7E) -> float64 values."""
    code = np.asarray(code, dtype=np.int64)
    e = (code >> 3) & 15
    m = code & 7
    val = np.where(e == 0, m * 2.0 ** -9, (8 + m) * np.ldexp(1.0, e - 10))
    return np.where((code & 0x7F) == 0x7F, np.nan, val)


def e8m0_decode(code):
    """E8M0 codes -> float64 values 2**(code-127)."""
    code = np.asarray(code, dtype=np.int64)
    return np.where(code == 255, np.nan, np.ldexp(1.0, code - 127))


def floor_log2(a):
    """floor(log2 a) for positive finite values (exact, via the exponent)."""
    _, e2 = np.frexp(np.asarray(a, dtype=np.float64))
    return e2.astype(np.int64) - 1


# --------------------------------------------------------------------------
# quantizer
# --------------------------------------------------------------------------

class FP4Tensor:
    """One quantized matrix in outer x inner form (blocks along inner)."""

    def __init__(self, fmt, outer, inner, codes, scales, tensor_scale):
        self.fmt = fmt                    # "mx" or "nv"
        self.outer = outer
        self.inner = inner
        self.codes = codes                # outer x inner uint8 nibble codes
        self.scales = scales              # outer x inner/bs uint8 scale codes
        self.tensor_scale = tensor_scale  # float32 (NVFP4) or None

    @property
    def block(self):
        return MX_BLOCK if self.fmt == "mx" else NV_BLOCK

    @property
    def packed(self):
        return pack_codes(self.codes)

    @property
    def scales_tc(self):
        return swizzle_scales(self.scales, self.block)

    def scale_values(self):
        if self.fmt == "mx":
            return e8m0_decode(self.scales)
        return e4m3_decode(self.scales) * np.float64(self.tensor_scale)

    def dequantize(self):
        """float64 outer x inner values."""
        return dequantize(self.codes, self.scales, self.fmt, self.tensor_scale)

    def colsum(self):
        """Sum over the inner axis of the dequantized values (one per outer)."""
        return self.dequantize().sum(axis=1)


def dequantize(codes, scales, fmt, tensor_scale=None):
    """Decode nibble codes and per-block scale codes to float64."""
    bs = MX_BLOCK if fmt == "mx" else NV_BLOCK
    outer, inner = codes.shape
    vals = e2m1_decode(codes).reshape(outer, inner // bs, bs)
    if fmt == "mx":
        sv = e8m0_decode(scales)
    else:
        sv = e4m3_decode(scales) * np.float64(tensor_scale)
    return (vals * sv[:, :, None]).reshape(outer, inner)


def nv_tensor_scale(alpha):
    """NVFP4 tensor scale s_t = alpha / 2688 in float32 (1 when alpha == 0)."""
    alpha = F32(alpha)
    if alpha == 0:
        return F32(1.0)
    return F32(alpha / NV_TENSOR_DIV)


def quantize(X, fmt, axis=1, tensor_amax=None):
    """Quantize a float32 matrix to FP4.

    X: 2-D float32 array (rows x cols).  ``axis=1`` puts blocks along the
    columns (outer = rows); ``axis=0`` puts blocks along the rows
    (outer = cols).  ``tensor_amax`` overrides the NVFP4 tensor maximum
    (default: max |X|).  Returns an FP4Tensor.
    """
    X = np.asarray(X)
    if X.dtype != F32:
        raise TypeError("quantizer input must be float32 (the GPU kernels see float32)")
    Z = X if axis == 1 else X.T
    outer, inner = Z.shape
    bs = MX_BLOCK if fmt == "mx" else NV_BLOCK
    if inner % bs:
        raise ValueError("blocked dimension must be a multiple of the block size")
    blocks = Z.reshape(outer, inner // bs, bs)
    amax = np.max(np.abs(blocks), axis=2)                     # float32, exact
    if fmt == "mx":
        se = np.where(amax == 0, -127, np.clip(floor_log2(np.where(amax == 0, 1, amax)) - 2, -127, 127))
        scales = (se + 127).astype(np.uint8)
        inv = np.ldexp(F32(1.0), (-se).astype(np.int32)).astype(F32)   # 2**-se, normal float32
        q = (blocks * inv[:, :, None]).astype(F32)
        codes = e2m1_encode(q)
        codes = np.where((amax == 0)[:, :, None], np.uint8(0), codes)
        return FP4Tensor("mx", outer, inner, codes.reshape(outer, inner), scales, None)
    if fmt != "nv":
        raise ValueError("fmt must be 'mx' or 'nv'")
    alpha = F32(np.max(np.abs(Z))) if tensor_amax is None else F32(tensor_amax)
    s_t = nv_tensor_scale(alpha)
    t = ((amax / s_t).astype(F32) / F32(6.0)).astype(F32)
    dcode = e4m3_encode(t)
    d = e4m3_decode(dcode).astype(F32)
    with np.errstate(divide="ignore", over="ignore", invalid="ignore"):
        enc = (F32(1.0) / (d * s_t).astype(F32)).astype(F32)
        q = (blocks * enc[:, :, None]).astype(F32)
    codes = e2m1_encode(q)
    codes = np.where((d == 0)[:, :, None], np.uint8(0), codes)
    return FP4Tensor("nv", outer, inner, codes.reshape(outer, inner), dcode, s_t)


# --------------------------------------------------------------------------
# storage layouts
# --------------------------------------------------------------------------

def pack_codes(codes):
    """outer x inner nibble codes -> outer x inner/2 bytes (even index low)."""
    codes = np.asarray(codes, dtype=np.uint8)
    return (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)


def unpack_codes(packed):
    packed = np.asarray(packed, dtype=np.uint8)
    out = np.empty((packed.shape[0], packed.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = packed & 0xF
    out[:, 1::2] = packed >> 4
    return out


def tc_scale_shape(outer, inner, bs):
    """(padded rows, padded scale columns) of the tensor-core scale layout."""
    rows = -(-outer // 128) * 128
    per_tile = KTILE // bs
    cols = -(-(inner // bs) // per_tile) * per_tile
    return rows, cols


def tc_scale_offset(r, c, padded_cols):
    """Byte offset of scale (row r, scale column c) in the tensor-core layout."""
    r = np.asarray(r, dtype=np.int64)
    c = np.asarray(c, dtype=np.int64)
    chunk = (r // 128) * (padded_cols // 4) + c // 4
    return chunk * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + (c % 4)


def swizzle_scales(scales, bs):
    """Linear outer x inner/bs scale codes -> flat tensor-core layout."""
    outer, nb = scales.shape
    rows, cols = tc_scale_shape(outer, nb * bs, bs)
    out = np.zeros(rows * cols, dtype=np.uint8)
    r, c = np.meshgrid(np.arange(outer), np.arange(nb), indexing="ij")
    out[tc_scale_offset(r, c, cols)] = scales
    return out


def unswizzle_scales(flat, outer, inner, bs):
    """Flat tensor-core layout -> linear outer x inner/bs scale codes."""
    rows, cols = tc_scale_shape(outer, inner, bs)
    flat = np.asarray(flat, dtype=np.uint8)
    if flat.size != rows * cols:
        raise ValueError("scale buffer has the wrong size")
    nb = inner // bs
    r, c = np.meshgrid(np.arange(outer), np.arange(nb), indexing="ij")
    return flat[tc_scale_offset(r, c, cols)]


def from_storage(fmt, outer, inner, packed, scales_tc, tensor_scale=None):
    """Rebuild an FP4Tensor from stored bytes (packed codes + tensor-core scales)."""
    bs = MX_BLOCK if fmt == "mx" else NV_BLOCK
    codes = unpack_codes(np.asarray(packed, dtype=np.uint8).reshape(outer, inner // 2))
    scales = unswizzle_scales(scales_tc, outer, inner, bs)
    ts = None if fmt == "mx" else F32(tensor_scale)
    return FP4Tensor(fmt, outer, inner, codes, scales, ts)
