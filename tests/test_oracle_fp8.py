"""Pins for the oracle's E4M3 encoder.

The encoder (round to nearest even, saturate at 448) is compared with
  * a brute-force nearest-value search over all 127 positive codes, whose
    values come from the OCP E4M3 definition written out here;
  * PyTorch's CPU cast to float8_e4m3fn (after clamping to +-448, since that
    cast does not saturate);
over every finite bf16 bit pattern, every tie point between neighbours, and a
strided sweep of fp32 bit patterns.
"""
import numpy as np
import torch


def e4m3_value(code: int) -> float:
    """OCP E4M3: bias 7, 3 mantissa bits, subnormals m*2^-9, S.1111.111 = NaN."""
    s = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return s * m * 2.0 ** -9
    return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)


POS_CODES = np.arange(0x7F)                      # 0x00..0x7E, all finite non-negative
POS_VALUES = np.array([e4m3_value(int(c)) for c in POS_CODES])


def brute_force_encode(v: np.ndarray) -> np.ndarray:
    v = v.astype(np.float64)
    a = np.minimum(np.abs(v), 448.0)
    d = np.abs(a[:, None] - POS_VALUES[None, :])
    best = d.min(axis=1, keepdims=True)
    cand = d == best
    # among tied candidates prefer the even code (even mantissa)
    even = cand & (POS_CODES[None, :] % 2 == 0)
    pick = np.where(even.any(axis=1), even.argmax(axis=1), cand.argmax(axis=1))
    sign = np.signbit(v).astype(np.uint8) << 7
    return (POS_CODES[pick].astype(np.uint8) | sign).astype(np.uint8)


def all_finite_bf16_as_f32():
    bits = np.arange(1 << 16, dtype=np.uint32) << 16
    f = bits.view(np.float32)
    return f[np.isfinite(f)]


def test_known_codes(oracle_lib):
    enc = oracle_lib.e4m3_encode
    vals = np.array([1.0, -1.0, 448.0, -448.0, 1e9, -np.inf, np.inf, 2.0 ** -9, 2.0 ** -6,
                     0.0, -0.0, 2.0 ** -10, 1.5 * 2.0 ** -10, 464.0, 465.0], np.float32)
    want = [0x38, 0xB8, 0x7E, 0xFE, 0x7E, 0xFE, 0x7E, 0x01, 0x08, 0x00, 0x80, 0x00, 0x01, 0x7E, 0x7E]
    assert enc(vals).tolist() == want
    assert enc(np.array([np.nan], np.float32))[0] & 0x7F == 0x7F


def test_representable_values_round_trip(oracle_lib):
    for code in list(range(0x00, 0x7F)) + list(range(0x80, 0xFF)):
        v = np.array([e4m3_value(code)], np.float32)
        assert oracle_lib.e4m3_encode(v)[0] == code, hex(code)


def test_brute_force_all_bf16(oracle_lib):
    f = all_finite_bf16_as_f32()
    np.testing.assert_array_equal(oracle_lib.e4m3_encode(f), brute_force_encode(f))


def test_ties_and_neighbours(oracle_lib):
    mids = (POS_VALUES[:-1] + POS_VALUES[1:]) / 2.0          # exact in fp32
    m32 = mids.astype(np.float32)
    assert (m32.astype(np.float64) == mids).all()
    up = np.nextafter(m32, np.float32(np.inf))
    dn = np.nextafter(m32, np.float32(0))
    f = np.concatenate([m32, up, dn, -m32, -up, -dn])
    np.testing.assert_array_equal(oracle_lib.e4m3_encode(f), brute_force_encode(f))
    # ties go to the even code
    codes = oracle_lib.e4m3_encode(m32)
    assert (codes % 2 == 0).all()


def _torch_cast(f: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(f.astype(np.float32)).clamp(-448.0, 448.0)
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_against_torch_cast(oracle_lib):
    f = all_finite_bf16_as_f32()
    np.testing.assert_array_equal(oracle_lib.e4m3_encode(f), _torch_cast(f))
    bits = np.arange(0, 1 << 32, 4099, dtype=np.uint64).astype(np.uint32)
    g = bits.view(np.float32)
    g = g[np.isfinite(g)]
    np.testing.assert_array_equal(oracle_lib.e4m3_encode(g), _torch_cast(g))
    rng = np.random.default_rng(7)
    h = (rng.standard_normal(1 << 20) * rng.choice([1e-3, 1.0, 64.0, 500.0], 1 << 20)).astype(np.float32)
    np.testing.assert_array_equal(oracle_lib.e4m3_encode(h), _torch_cast(h))
