"""CPU checks of the arithmetic the int8 kernels use in place of the plain
definition, over the whole bf16 domain.

The quantising kernel does not divide every element: it multiplies by the
correctly rounded reciprocal of the channel scale, rounds by adding
1.5 * 2^23, and takes the exact IEEE quotient only where the product lies
within 2^-13 of a half-integer (a band containing every |t| * 2^-20
distance, since |t| <= 127 (1 + 2^-23)).  The dequantising kernel turns a code
byte into a float by placing it in the mantissa of 1.5 * 2^23.  These tests
emulate those steps in NumPy float32 and require them to equal the oracle's
definition (rint of the IEEE quotient; the int8 value) for every bf16 input
of a block against its absmax, so the shortcut is pinned independently of
the GPU."""
import numpy as np

from oracle.quant import quantize_block

F32 = np.float32
K_ROUND = F32(12582912.0)          # 1.5 * 2^23


def _bf16_bits_upto(a_bits):
    """All non-negative bf16 bit patterns <= a (finite), as uint16."""
    return np.arange(0, int(a_bits) + 1, dtype=np.uint32).astype(np.uint16)


def _f32(bits16):
    return (bits16.astype(np.uint32) << 16).view(np.float32)


def _kernel_rule(x, a):
    """The quantising kernel's per-element code for values x (float32) of a
    channel whose absmax is a (float32 scalar)."""
    sc = F32(a / F32(127.0))
    usable = F32(2.0 ** -100) <= sc <= F32(2.0 ** 100)
    rc = F32(F32(1.0) / sc) if usable else F32(0.0)
    with np.errstate(over="ignore", invalid="ignore"):
        t = (x * rc).astype(np.float32)
        y = (t + K_ROUND).astype(np.float32)
        r = (y - K_ROUND).astype(np.float32)
        e = (t - r).astype(np.float32)
    # |t - rint(t)| > 1/2 - 2^-13
    near = (np.abs(e) > F32(0.5 - 2.0 ** -13)) | (not usable and sc != 0)
    code = (y.view(np.uint32) & 0xFF).astype(np.uint8).view(np.int8).astype(np.int32)
    if near.any():
        with np.errstate(divide="ignore", invalid="ignore"):
            q = (x[near] / sc).astype(np.float32) if sc != 0 else np.zeros(int(near.sum()), np.float32)
        code[near] = np.rint(q).astype(np.int32)
    return code, int(near.sum())


def _check_absmax(a_bits):
    pos = _bf16_bits_upto(a_bits)
    col = np.concatenate([pos, pos | np.uint16(0x8000)])     # every bf16 x with |x| <= a, both signs
    ref_codes, ref_a = quantize_block(col.reshape(-1, 1))
    a = _f32(np.array([a_bits], dtype=np.uint16))[0]
    assert ref_a[0] == a
    got, n_near = _kernel_rule(_f32(col), a)
    assert np.array_equal(got, ref_codes[:, 0].astype(np.int32)), hex(int(a_bits))
    return n_near, col.size


def test_product_rule_equals_ieee_quotient_for_every_bf16_input():
    near = total = 0
    # every absmax mantissa at three binades where the reciprocal is used (the
    # rule is exact under scaling by 2^k); each block holds every bf16 |x| <= a
    for e_bits in (0x3F80, 0x2000, 0x5F00):
        for m in range(128):
            n, t = _check_absmax(e_bits | m)
            near += n
            total += t
    # exact ties exist (x = a / 2, absmax mantissa 254/128), so the fallback is
    # exercised, on a small share of the inputs
    assert 0 < near < total // 50


def test_product_rule_degenerate_absmax():
    _check_absmax(0x0000)       # all-zero channel: codes 0
    _check_absmax(0x0001)       # smallest subnormal absmax: scale below 2^-100, always divides
    _check_absmax(0x0080)       # smallest normal
    _check_absmax(0x7F7F)       # largest finite bf16


def test_round_by_adding_one_point_five_two_to_the_23():
    t = np.concatenate([np.linspace(-127.49, 127.49, 100001, dtype=np.float32),
                        np.array([0.5, 1.5, 2.5, -0.5, -1.5, 63.5, -63.5, -0.0], dtype=np.float32)])
    y = (t + K_ROUND).astype(np.float32)
    assert np.array_equal((y - K_ROUND).astype(np.float32), np.rint(t))       # ties to even
    low = (y.view(np.uint32) & 0xFF).astype(np.uint8).view(np.int8)
    assert np.array_equal(low.astype(np.int32), np.rint(t).astype(np.int32))


def _byte_perm(x, y, s):
    b = [(x >> (8 * i)) & 0xFF for i in range(4)] + [(y >> (8 * i)) & 0xFF for i in range(4)]
    return sum(b[(s >> (4 * i)) & 0x7] << (8 * i) for i in range(4))


def test_code_byte_to_float_by_mantissa_placement():
    for k in range(-128, 128):
        for pos in range(4):
            w = ((k & 0xFF) << (8 * pos)) | (0x3C << (8 * ((pos + 1) % 4)))
            bits = _byte_perm(w ^ 0x80808080, 0x4B400000, 0x7640 | pos)
            v = F32(np.array([bits], dtype=np.uint32).view(np.float32)[0] - F32(12583040.0))
            assert v == F32(k)


# ---- the same rule with the 4- and 3-bit scales
# The kernels use one code path for every width: t = RN(x * RN(1 / sc)),
# y = RN(t + 1.5 * 2^23), the exact quotient where |t - rint(t)| > 1/2 - 2^-13,
# and the field taken from the low bits of y's pattern plus the bias (8 or 4).
# With sc = bf16(a / 7) or bf16(a / 3) the band still holds every element whose
# product may round differently (|t| < 7.03 resp. 3.02).

def _bf16_round(x):
    """fp32 -> fp32 value of its bf16 rounding (nearest, ties to even)."""
    b = np.asarray(x, dtype=np.float32).reshape(-1).view(np.uint32).astype(np.uint64)
    r = ((b + 0x7FFF + ((b >> 16) & 1)) >> 16) << 16
    return r.astype(np.uint32).view(np.float32).reshape(np.shape(x))


def _kernel_rule_packed(x, a, bits):
    qmax, bias, mask = (7, 8, 0xF) if bits == 4 else (3, 4, 0x7)
    sc = F32(_bf16_round(F32(a / F32(qmax))))
    usable = F32(2.0 ** -100) <= sc <= F32(2.0 ** 100)
    rc = F32(F32(1.0) / sc) if usable else F32(0.0)
    with np.errstate(over="ignore", invalid="ignore"):
        t = (x * rc).astype(np.float32)
        y = (t + K_ROUND).astype(np.float32)
        r = (y - K_ROUND).astype(np.float32)
        e = (t - r).astype(np.float32)
    near = (np.abs(e) > F32(0.5 - 2.0 ** -13)) | (not usable and sc != 0)
    if near.any():
        with np.errstate(divide="ignore", invalid="ignore"):
            q = (x[near] / sc).astype(np.float32) if sc != 0 else np.zeros(int(near.sum()), np.float32)
        y[near] = (q + K_ROUND).astype(np.float32)
    field = (y.view(np.uint32) + np.uint32(bias)) & np.uint32(mask)
    return field.astype(np.int32) - bias, int(near.sum())


def _check_absmax_packed(a_bits, bits):
    from oracle.quant import quantize_block_int3, quantize_block_int4
    pos = _bf16_bits_upto(a_bits)
    col = np.concatenate([pos, pos | np.uint16(0x8000)])
    ref_codes, _ = (quantize_block_int4 if bits == 4 else quantize_block_int3)(col.reshape(-1, 1))
    a = _f32(np.array([a_bits], dtype=np.uint16))[0]
    got, n_near = _kernel_rule_packed(_f32(col), a, bits)
    assert np.array_equal(got, ref_codes[:, 0].astype(np.int32)), (bits, hex(int(a_bits)))
    return n_near, col.size


def test_product_rule_equals_ieee_quotient_packed_widths():
    for bits in (4, 3):
        near = total = 0
        for e_bits in (0x3F80, 0x2000, 0x5F00):
            for m in range(128):
                n, t = _check_absmax_packed(e_bits | m, bits)
                near += n
                total += t
        assert 0 < near < total // 20, bits    # ties x = s * (k + 1/2) exist and take the exact path
        for a_bits in (0x0000, 0x0001, 0x0080, 0x7F7F):
            _check_absmax_packed(a_bits, bits)
