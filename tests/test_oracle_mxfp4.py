"""Pins for the MXFP4 weight format (OCP Microscaling v1.0, e2m1 values with one
e8m0 scale per 32 along K), used for the routed experts' weights."""
import numpy as np
import torch

import oracle
import workloads

# e2m1: sign bit, 2 exponent bits (bias 1), 1 mantissa bit; written out from the format
E2M1 = {0: 0.0, 1: 0.5, 2: 1.0, 3: 1.5, 4: 2.0, 5: 3.0, 6: 4.0, 7: 6.0}


def _e2m1_from_bits(c):
    s = -1.0 if c & 8 else 1.0
    e = (c >> 1) & 3
    m = c & 1
    if e == 0:                       # subnormal: m * 2^(1-1) * 0.5
        return s * m * 0.5
    return s * (1.0 + m / 2.0) * 2.0 ** (e - 1)


def test_code_table_from_bit_fields():
    for c in range(16):
        v = _e2m1_from_bits(c)
        assert abs(v) == E2M1[c & 7]
        assert (v < 0) == (bool(c & 8) and (c & 7) != 0)


def test_dequantize_every_code_and_scale():
    for sbyte in (127, 120, 134, 1):
        codes = np.zeros((1, 16), np.uint8)
        for j in range(32):          # element j holds code j % 16
            c = j % 16
            if j % 2 == 0:
                codes[0, j // 2] |= c
            else:
                codes[0, j // 2] |= c << 4
        scales = np.array([[sbyte]], np.uint8)
        v = oracle.mxfp4_dequantize(codes, scales)
        expect = np.array([_e2m1_from_bits(j % 16) * 2.0 ** (sbyte - 127) for j in range(32)])
        assert np.array_equal(v[0], expect)


def test_nibble_order_low_first():
    v = oracle.mxfp4_dequantize(np.array([[0x21] + [0] * 15], np.uint8), np.array([[127]], np.uint8))
    assert v[0, 0] == 0.5 and v[0, 1] == 1.0


def test_pack_roundtrip_exact_values():
    rng = np.random.default_rng(1)
    mags = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)
    vals = mags[rng.integers(0, 8, (16, 64))] * np.where(rng.random((16, 64)) < 0.5, -1, 1)
    vals[:, ::32] = 6.0                       # every block reaches amax 6 -> X = 0 exactly
    X = rng.integers(-20, 20, (16, 2))
    w = vals * np.repeat(2.0 ** X, 32, axis=1)
    q, sc = workloads.mxfp4_pack(torch.from_numpy(w.astype(np.float32)))
    back = oracle.mxfp4_dequantize(q.numpy(), sc.numpy())
    assert np.array_equal(back, w)


def test_pack_error_bound_gaussian():
    g = torch.Generator().manual_seed(3)
    w = torch.randn(64, 256, generator=g) / 16
    q, sc = workloads.mxfp4_pack(w)
    back = oracle.mxfp4_dequantize(q.numpy(), sc.numpy())
    w64 = w.double().numpy()
    blk = np.abs(w64).reshape(64, 8, 32).max(-1)
    scale = np.repeat(2.0 ** (np.floor(np.log2(blk)) - 2), 32, axis=1)
    # nearest e2m1 point; above 6 (up to 8 in scaled units) values saturate to 6
    assert np.all(np.abs(back - w64) <= scale * 2.0 + 1e-12)
    # below the saturation region the error is at most half a spacing of 0.5 or 1
    small = np.abs(w64) / scale < 4
    assert np.all(np.abs(back - w64)[small] <= scale[small] * 0.5 + 1e-12)
