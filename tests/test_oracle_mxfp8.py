"""Pins for the oracle's MXFP8 activation quantisation (reading R15 of the
block-scaled variant: OCP Microscaling v1.0, e4m3 elements, e8m0 scale per 32
along the contraction). Each check is against the format's definition, brute
force over all codes, or a closed form, never a retyped formula."""
import math
import struct

import numpy as np
import pytest

import oracle
import workloads


def _finite_codes():
    c = np.arange(256, dtype=np.uint8)
    return c[(c & 0x7F) != 0x7F]


def test_e4m3_landmarks():
    d = oracle.e4m3_decode(np.array([0x00, 0x80, 0x38, 0xB8, 0x7E, 0xFE, 0x01, 0x08, 0x07, 0x30, 0x40],
                                    dtype=np.uint8))
    expect = [0.0, -0.0, 1.0, -1.0, 448.0, -448.0, 2.0 ** -9, 2.0 ** -6, 7 * 2.0 ** -9, 0.5, 2.0]
    assert list(d) == expect
    assert np.signbit(d[1])
    assert np.isnan(oracle.e4m3_decode(np.array([0x7F, 0xFF], dtype=np.uint8))).all()


def test_e4m3_values_are_distinct_and_ordered():
    pos = oracle.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    assert np.all(np.diff(pos) > 0)                       # codes 0..126 increase strictly
    assert pos.size == 127 and pos[-1] == oracle.E4M3_MAX
    # each binade above the subnormals has 8 values spaced 2^(e-10)
    for e in range(1, 16):
        vals = pos[(e << 3):(e << 3) + 8]
        vals = vals[~np.isnan(vals)]
        assert np.allclose(np.diff(vals), 2.0 ** (e - 10), rtol=0, atol=0)


def test_e4m3_encode_inverts_decode():
    c = _finite_codes()
    v = oracle.e4m3_decode(c)
    v = np.where(c == 0x80, -0.0, v)
    assert np.array_equal(oracle.e4m3_encode(v), c)


def test_e4m3_encode_is_nearest_with_ties_to_even():
    rng = np.random.default_rng(1)
    table_codes = _finite_codes()
    table = oracle.e4m3_decode(table_codes)
    v = np.concatenate([rng.uniform(-450, 450, 3000), rng.uniform(-1, 1, 3000) * 2.0 ** -6,
                        # exact midpoints between neighbours
                        (table[1:126] + table[2:127]) / 2])
    code = oracle.e4m3_encode(v)
    got = oracle.e4m3_decode(code)
    for x, c, g in zip(v, code, got):
        dist = np.abs(table - min(abs(x), 448.0) * math.copysign(1, x))
        best = dist.min()
        assert abs(abs(g) - min(abs(x), 448.0)) == pytest.approx(best, abs=0)
        ties = table_codes[dist == best]
        if len(set(np.abs(oracle.e4m3_decode(ties)))) > 1:   # a real tie between two values
            assert (c & 1) == 0


def test_e4m3_saturates():
    assert list(oracle.e4m3_encode(np.array([448.0, 449.0, 464.0, 1e6, -500.0]))) == [0x7E, 0x7E, 0x7E,
                                                                                    0x7E, 0xFE]


def test_mxfp8_scale_closed_form():
    rng = np.random.default_rng(2)
    v = rng.standard_normal((7, 96)) * np.exp2(rng.integers(-20, 20, size=(7, 1)))
    codes, scales = oracle.mxfp8_quantize(v)
    amax = np.abs(v.reshape(7, 3, 32)).max(axis=-1)
    assert np.array_equal(scales.astype(int), np.floor(np.log2(amax)).astype(int) + 119)
    # every scaled element fits the e4m3 range: |v| / 2^(byte-127) < 2^9, and all codes are finite
    assert not np.isnan(oracle.e4m3_decode(codes)).any()


def test_mxfp8_is_nearest_grid_point():
    rng = np.random.default_rng(3)
    v = rng.standard_normal((4, 64))
    codes, scales = oracle.mxfp8_quantize(v)
    dq = oracle.mxfp8_dequantize(codes, scales)
    table = oracle.e4m3_decode(_finite_codes())
    for r in range(4):
        for k in range(64):
            X = 2.0 ** (int(scales[r, k // 32]) - 127)
            grid = table * X
            assert abs(dq[r, k] - v[r, k]) == pytest.approx(np.abs(grid - v[r, k]).min(), abs=0)


def test_mxfp8_exact_on_representable_blocks():
    # e4m3 values times 2^-10 whose largest lies in [256, 448] * 2^-10: the scale is then
    # exactly 2^-10 and every element is back on the e4m3 grid
    rng = np.random.default_rng(4)
    codes_in = rng.integers(0, 0x7F, size=(3, 64)).astype(np.uint8)
    codes_in[:, 7] = 0x7A                         # 320: floor(log2) = 8 in each first block
    codes_in[:, 40] = 0x79                        # 288 in each second block
    codes_in[1] |= 0x80                           # a negative row
    v = oracle.e4m3_decode(codes_in) * 2.0 ** -10
    codes, scales = oracle.mxfp8_quantize(v)
    assert (scales == 117).all()                  # 8 - 8 - 10 + 127
    assert np.array_equal(codes, codes_in)
    assert np.array_equal(oracle.mxfp8_dequantize(codes, scales), v)


def test_mxfp8_zero_and_saturating_blocks():
    codes, scales = oracle.mxfp8_quantize(np.zeros((1, 32)))
    assert scales[0, 0] == 0 and not codes.any()
    # amax 500: scale 2^(8-8) = 1, and 500 saturates to 448 (the OCP rule for e4m3)
    v = np.zeros((1, 32))
    v[0, 5] = 500.0
    v[0, 6] = -300.0
    codes, scales = oracle.mxfp8_quantize(v)
    assert scales[0, 0] == 127
    dq = oracle.mxfp8_dequantize(codes, scales)
    assert dq[0, 5] == 448.0 and dq[0, 6] == -288.0          # 300 -> nearest of 288 / 320: 288


def test_mxfp8_blocks_follow_the_last_axis():
    # two rows with very different magnitudes keep their own scales
    v = np.ones((2, 32))
    v[1] *= 1024.0
    _, scales = oracle.mxfp8_quantize(v)
    assert scales[0, 0] == 119 and scales[1, 0] == 129


def test_block_scaled_layer_close_to_bf16_layer():
    """R15 changes only the routed activations' rounding: on the tiny
    block-scaled config the output stays close to the same layer with bf16
    activations (e4m3 keeps 3 mantissa bits: a relative rounding error of at
    most 2^-4 per element, a few percent of RMS after the dot products) and
    differs from it (the quantisation ran)."""
    cfg = workloads.CONFIGS["tiny_a8"]
    d = workloads.generate(cfg, "cpu", T=24)
    from helpers import experts_of, host_inputs
    h = host_inputs(d)
    ex = experts_of(d)
    a8 = oracle.layer_forward(cfg, h["x"], h["Wr"], h["bias"], ex, h["Wg_s"], h["Wu_s"], h["Wd_s"])
    b16 = oracle.layer_forward(cfg.with_(wfmt=workloads.MOE_W_MXFP4), h["x"], h["Wr"], h["bias"], ex,
                               h["Wg_s"], h["Wu_s"], h["Wd_s"])
    diff = a8["y_f32"] - b16["y_f32"]
    rms = np.sqrt(np.mean(b16["y_f32"].astype(np.float64) ** 2))
    assert 0 < np.abs(diff).max() < 0.4 * rms
    assert np.sqrt(np.mean(diff.astype(np.float64) ** 2)) < 0.08 * rms


# ---------------------------------------------------------------- one token, pure Python

def _py_e4m3_values():
    """(code, value) of the 127 non-negative finite e4m3 codes from the bit
    fields: exponent bits 6..3 (bias 7), mantissa bits 2..0, exponent 0
    subnormal."""
    out = []
    for c in range(0x7F):
        e, m = c >> 3, c & 7
        out.append((c, (m / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7)))
    return out


_PY_E4M3 = _py_e4m3_values()


def _py_mx_block(vals):
    """MXFP8 value of each element of one 32-element block (R15), by linear
    search over the e4m3 values: scale 2^(floor(log2 amax) - 8) with its byte
    clamped to [0, 254]; nearest value, ties to the even code, saturation at
    448; the sign kept."""
    amax = max(abs(v) for v in vals)
    if amax == 0.0:
        byte = 0
    else:
        _, ex = math.frexp(amax)                 # amax = f * 2^ex, f in [0.5, 1)
        byte = min(max(ex - 1 - 8 + 127, 0), 254)
    X = 2.0 ** (byte - 127)
    out = []
    for v in vals:
        a = min(abs(v) / X, 448.0)
        best = None
        for c, q in _PY_E4M3:
            key = (abs(q - a), c & 1)            # nearer first, then the even code
            if best is None or key < best[0]:
                best = (key, q)
        out.append(math.copysign(best[1] * X, v))
    return out


def _py_mx(row):
    return [q for b in range(0, len(row), 32) for q in _py_mx_block(row[b:b + 32])]


def _f32(v):
    return struct.unpack("<f", struct.pack("<f", v))[0]


def _py_bf16(v):
    (u,) = struct.unpack("<I", struct.pack("<f", v))
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return struct.unpack("<f", struct.pack("<I", u << 16))[0]


def _py_swiglu(xrow, Wg, Wu, Wd, L, h_round):
    I, H = Wg.shape
    a = []
    for i in range(I):
        g = _f32(math.fsum(xrow[k] * Wg[i, k] for k in range(H)))
        u = _f32(math.fsum(xrow[k] * Wu[i, k] for k in range(H)))
        if L > 0:
            g, u = min(max(g, -L), L), min(max(u, -L), L)
        a.append(_f32(g / (1.0 + math.exp(-g)) * u))
    h = h_round(a)
    return [_f32(math.fsum(h[i] * Wd[n, i] for i in range(I))) for n in range(Wd.shape[0])]


@pytest.mark.parametrize("t", [5])
def test_block_scaled_layer_one_token_pure_python(t):
    """One token of the tiny block-scaled layer from explicit loops: x and the
    fp32 h of every routed slot quantised to MXFP8 by linear search over the
    e4m3 values, MXFP4 weights at their exact values, exact dot products
    (fsum) rounded to fp32, y_slot = w * o, fp32 sum in slot order; the shared
    expert on bf16 x with a bf16 h. Equal bit for bit to layer_forward."""
    from helpers import experts_of, host_inputs
    cfg = workloads.CONFIGS["tiny_a8"]
    d = workloads.generate(cfg, "cpu", T=8)
    h = host_inputs(d)
    ex = experts_of(d)
    out = oracle.layer_forward(cfg, h["x"], h["Wr"], h["bias"], ex, h["Wg_s"], h["Wu_s"], h["Wd_s"])
    f = oracle.bf16_bits_to_f64
    xr = f(h["x"][t]).tolist()
    xq = _py_mx(xr)
    assert xq != xr                                   # the quantisation changes x
    acc = None
    for k in range(cfg.K):
        e = int(out["idx"][t, k])
        Wg, Wu, Wd = ex(e)
        o = _py_swiglu(xq, Wg, Wu, Wd, cfg.limit_routed, _py_mx)
        wk = float(out["w"][t, k])
        contrib = [_f32(wk * v) for v in o]
        acc = contrib if acc is None else [_f32(a + c) for a, c in zip(acc, contrib)]
    osh = _py_swiglu(xr, f(h["Wg_s"]), f(h["Wu_s"]), f(h["Wd_s"]), cfg.limit_shared,
                     lambda a: [_py_bf16(v) for v in a])
    y32 = [_f32(a + c) for a, c in zip(acc, osh)]
    assert np.array_equal(out["y_f32"][t], np.array(y32, np.float32))
    assert np.array_equal(f(out["y"][t]), np.array([_py_bf16(v) for v in y32]))
