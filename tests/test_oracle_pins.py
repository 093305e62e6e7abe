"""Pins of the oracle against what the pages and the mathematics fix.

Each test checks one oracle function against something other than itself:
the pages' numbers (6.75 MB per expert), hand-derived byte images, closed
forms, special cases that reduce to a textbook or library routine, and brute
force. A plausible mistake (a dropped bias term, a wrong group index, a
transposed operand, a swapped gate/up, a reversed sort or tie-break) fails at
least one of them. All CPU-only.
"""
import math
import os

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield line


def _bf16(v):
    """bf16 bits of a float that is exactly representable in bf16."""
    b = np.float32(v).view(np.uint32)
    assert (b & 0xFFFF) == 0, v
    return np.uint16(b >> 16)


def _rand_layer(rng, rows, cols, bits, group):
    codes = rng.integers(0, 1 << bits, size=(rows, cols), dtype=np.uint8)
    # scale/bias as bf16 by truncating random fp32 bit patterns
    s32 = rng.uniform(0.005, 0.02, size=(rows, cols // group)).astype(np.float32).view(np.uint32)
    b32 = rng.normal(0, 0.01, size=(rows, cols // group)).astype(np.float32).view(np.uint32)
    scale = (s32 >> 16).astype(np.uint16)
    bias = (b32 >> 16).astype(np.uint16)
    return codes, scale, bias


def _f64(bits):
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# ---- sizes (the page's 6.75 MB per expert) ----------------------------------

def test_expert_bytes_match_page(ref):
    for line in _rows("expert_bytes.txt"):
        H, I, bits, group, nbytes = map(int, line.split())
        assert ref.expert_bytes(H, I, bits, group) == nbytes
    assert ref.expert_bytes(4096, 1024, 4, 64) == int(6.75 * 2 ** 20)


# ---- bf16 conversions -------------------------------------------------------

def test_bf16_widening_exact(ref):
    assert ref.bf16_to_f64(0x3F80)[0] == 1.0
    assert ref.bf16_to_f64(0x4049)[0] == 3.140625
    assert ref.bf16_to_f64(0xC2F7)[0] == -123.5
    assert ref.bf16_to_f64(0x0001)[0] == 2.0 ** -133


def test_bf16_rounding_nearest_even(ref):
    cases = {
        1.0 + 2 ** -8: 0x3F80,               # tie, even stays 1.0
        1.0 + 3 * 2 ** -8: 0x3F82,           # tie, rounds to even 1+2^-6
        1.0 + 2 ** -8 + 2 ** -20: 0x3F81,    # above the tie
        -2.0: 0xC000,
        2.0 ** -133: 0x0001,                 # smallest subnormal
        1.5 * 2.0 ** -133: 0x0002,           # subnormal tie to even
        2.0 ** -134: 0x0000,                 # tie to even zero
        1e39: 0x7F80,                        # overflow
        0.0: 0x0000,
    }
    for v, bits in cases.items():
        assert int(ref.f64_to_bf16(v)[0]) == bits, (v, hex(bits))


# ---- packing ----------------------------------------------------------------

def test_pack_golden_bytes(ref):
    n = 0
    for line in _rows("pack_bytes.txt"):
        bits, group, codes, expect = [t.strip() for t in line.split("|")]
        bits, group = int(bits), int(group)
        c = np.array([[int(ch, 16) for ch in codes]], dtype=np.uint8)
        ng = c.shape[1] // group
        packed, sb = ref.pack(c, np.full((1, ng), 0x3F80, np.uint16), np.full((1, ng), 0xBF80, np.uint16),
                              bits, group)
        assert [int(v) for v in packed[0]] == [int(t, 16) for t in expect.split()]
        assert sb.shape == (1, ng, 2)
        assert (sb[..., 0] == 0x3F80).all() and (sb[..., 1] == 0xBF80).all()  # scale first
        n += 1
    assert n >= 6


@pytest.mark.parametrize("bits,group", [(4, 32), (4, 64), (2, 32), (2, 64), (4, 128), (3, 64), (3, 128)])
def test_pack_is_little_endian_bitstring(ref, bits, group):
    """Independent reading of the layout: a packed row is the row's codes
    written as one little-endian integer, sum_c q_c * 2^(c*bits)."""
    rng = np.random.default_rng(bits * 1000 + group)
    codes, scale, bias = _rand_layer(rng, 3, 256, bits, group)
    packed, sb = ref.pack(codes, scale, bias, bits, group)
    for r in range(3):
        big = sum(int(q) << (c * bits) for c, q in enumerate(codes[r]))
        assert bytes(packed[r]) == big.to_bytes(256 * bits // 8, "little")
        assert (sb[r, :, 0] == scale[r]).all() and (sb[r, :, 1] == bias[r]).all()


@pytest.mark.parametrize("bits,group", [(4, 32), (2, 64), (3, 64)])
def test_pack_roundtrip_and_range(ref, bits, group):
    rng = np.random.default_rng(7)
    codes, scale, bias = _rand_layer(rng, 5, 128, bits, group)
    packed, sb = ref.pack(codes, scale, bias, bits, group)
    c2, s2, b2 = ref.unpack(packed, sb, 5, 128, bits, group)
    assert (c2 == codes).all() and (s2 == scale).all() and (b2 == bias).all()
    codes[2, 3] = 1 << bits
    with pytest.raises(ValueError):
        ref.pack(codes, scale, bias, bits, group)


# ---- quantisation (weights -> codes, scale, bias) -----------------------------

def _bf16_round(v):
    """float value of the nearest bf16 (ties to even), via _rne_bf16_bits."""
    return float(_f64(np.array([_rne_bf16_bits(float(v))], np.uint16))[0])


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_quantize_constant_groups(ref, bits):
    """A constant group has range 0: scale 0, bias = bf16(the constant),
    every code 0."""
    w = np.array([[0.3] * 64 + [-2.5] * 64], np.float32)
    codes, scale, bias = ref.quantize(w, bits, 64)
    assert (codes == 0).all() and (scale == 0).all()
    assert [int(b) for b in bias[0]] == [_rne_bf16_bits(float(np.float32(0.3))), _rne_bf16_bits(-2.5)]


@pytest.mark.parametrize("bits,group", [(2, 64), (3, 64), (4, 64), (3, 128)])
def test_quantize_ramp_recovers_its_levels(ref, bits, group):
    """A group whose values are the 2^bits evenly spaced levels lo + j*d
    (bf16-exact, arithmetic exact in fp32) gets scale d, bias lo and code j
    for level j, so dequantisation returns every input exactly."""
    n = 1 << bits
    lo, d = -1.0, 0.25
    j = np.arange(group) % n
    w = (lo + j * d).astype(np.float32)[None, :]
    codes, scale, bias = ref.quantize(w, bits, group)
    assert (codes[0] == j).all()
    assert _f64(scale)[0, 0] == d and _f64(bias)[0, 0] == lo
    assert (codes[0] * d + lo == w[0]).all()


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_quantize_picks_the_nearest_level(ref, bits):
    """Brute force: each code is the nearest of the 2^bits levels bias + q*scale
    of its group (exact fp64 distances; inputs within 1e-4 of a midpoint
    between levels are left out, since the rounding of the kernel's binary32
    quotient decides those), and the round-trip error stays within half a
    scale step plus the bf16 rounding of scale and bias."""
    rng = np.random.default_rng(bits)
    G = 64
    w = (rng.normal(size=(6, 256)) * rng.uniform(0.01, 3.0, size=(6, 1))).astype(np.float32)
    # groups far from zero for their range: bf16(bias) misses the minimum by
    # up to a quarter, so codes clamp at the top or the bottom
    far = (rng.choice([-1.0, 1.0], size=(4, 1)) * rng.uniform(90.0, 120.0, size=(4, 1)) +
           rng.uniform(0.0, 1.0, size=(4, 256))).astype(np.float32)
    w = np.concatenate([w, far])
    codes, scale, bias = ref.quantize(w, bits, G)
    n = (1 << bits) - 1
    checked = 0
    for r in range(w.shape[0]):
        for g in range(w.shape[1] // G):
            wg = w[r, g * G:(g + 1) * G].astype(np.float64)
            lo, hi = wg.min(), wg.max()
            s_exact = (hi - lo) / n
            sh = _f64(scale[r, g])
            bh = _f64(bias[r, g])
            assert sh == _bf16_round(np.float32(np.float32(hi - lo) / np.float32(n)))
            assert bh == _bf16_round(lo)
            levels = bh + sh * np.arange(n + 1)
            for jj, v in enumerate(wg):
                q = int(codes[r, g * G + jj])
                t = (v - bh) / sh
                if abs(t - np.floor(t) - 0.5) < 1e-4:
                    continue
                assert q == int(np.argmin(np.abs(levels - v))), (r, g, jj)
                checked += 1
            err = np.abs(wg - (codes[r, g * G:(g + 1) * G] * sh + bh)).max()
            assert err <= sh / 2 + abs(bh - lo) + n * abs(sh - s_exact) + 1e-6 * max(abs(lo), abs(hi))
    assert checked >= 0.99 * w.size


def test_quantize_rejects_non_finite(ref):
    w = np.zeros((1, 64), np.float32)
    w[0, 5] = np.nan
    with pytest.raises(ValueError):
        ref.quantize(w, 4, 64)


# ---- dequant mat-vec --------------------------------------------------------

@pytest.mark.parametrize("bits,group", [(4, 32), (4, 64), (2, 64)])
def test_gemv_fma_rearrangement_identity(ref, bits, group):
    """The Flash-MoE page's identity: (q*s+b)*x == fma(q, s*x, b*x), and its
    per-group sum s*sum(qx) + b*sum(x): three forms agree to 1e-12."""
    rng = np.random.default_rng(11)
    codes, scale, bias = _rand_layer(rng, 64, 512, bits, group)
    x = rng.normal(size=512)
    y0 = ref.dequant_gemv(codes, scale, bias, group, x)
    y1 = ref.dequant_gemv_fma(codes, scale, bias, group, x)
    y2 = ref.dequant_gemv_grouped(codes, scale, bias, group, x)
    tol = 1e-12 * np.abs(y0).max()
    assert np.abs(y1 - y0).max() <= tol and np.abs(y2 - y0).max() <= tol


def test_gemv_constant_codes_closed_form(ref):
    """All codes c, per-row constant scale and bias: y_r = (c*s_r + b_r) * sum(x)."""
    rows, cols, group = 6, 256, 64
    rng = np.random.default_rng(3)
    x = rng.normal(size=cols)
    svals = [0.0078125, 0.015625, 0.01171875, 0.009765625, 0.005859375, 0.0185546875]
    bvals = [0.25, -0.5, 0.0, 0.125, -0.0625, 1.0]
    for c in (0, 5, 15):
        codes = np.full((rows, cols), c, np.uint8)
        scale = np.array([[_bf16(s)] * (cols // group) for s in svals], np.uint16)
        bias = np.array([[_bf16(b)] * (cols // group) for b in bvals], np.uint16)
        y = ref.dequant_gemv(codes, scale, bias, group, x)
        expect = np.array([(c * s + b) for s, b in zip(svals, bvals)]) * math.fsum(x)
        assert np.allclose(y, expect, rtol=1e-12, atol=1e-12)


def test_gemv_zero_codes_leave_bias_term(ref):
    """q = 0: y_r = sum_g b_{r,g} * sum_{j in g} x_j (catches a dropped or
    misindexed bias term)."""
    rng = np.random.default_rng(5)
    codes, scale, bias = _rand_layer(rng, 8, 256, 4, 32)
    codes[:] = 0
    x = rng.normal(size=256)
    y = ref.dequant_gemv(codes, scale, bias, 32, x)
    expect = (_f64(bias) * x.reshape(8, 32).sum(axis=1)[None, :]).sum(axis=1)
    assert np.allclose(y, expect, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("bits,group", [(4, 32), (2, 64)])
def test_gemv_one_hot_recovers_dequantised_column(ref, bits, group):
    """x = e_j gives column j dequantised, q[r,j]*s[r,j//G] + b[r,j//G], exactly
    (catches a transposed operand or a wrong group index)."""
    rng = np.random.default_rng(9)
    rows, cols = 16, 256
    codes, scale, bias = _rand_layer(rng, rows, cols, bits, group)
    for j in (0, 1, group - 1, group, cols - 1, 77):
        x = np.zeros(cols)
        x[j] = 1.0
        y = ref.dequant_gemv(codes, scale, bias, group, x)
        expect = codes[:, j].astype(np.float64) * _f64(scale[:, j // group]) + _f64(bias[:, j // group])
        assert (y == expect).all()


def test_gemv_matches_dense_library_matmul(ref):
    """Against numpy's dense float64 mat-vec of the explicitly dequantised matrix."""
    rng = np.random.default_rng(13)
    codes, scale, bias = _rand_layer(rng, 40, 320, 4, 32)
    x = rng.normal(size=320)
    W = codes.astype(np.float64) * np.repeat(_f64(scale), 32, axis=1) + np.repeat(_f64(bias), 32, axis=1)
    assert np.allclose(ref.dequant_gemv(codes, scale, bias, 32, x), W @ x, rtol=1e-12, atol=1e-12)


# ---- router -----------------------------------------------------------------

def test_router_one_hot_rows(ref):
    """W_r row e = c_e * unit vector at pi(e): logit_e = c_e * x[pi(e)] exactly."""
    E, H = 8, 64
    rng = np.random.default_rng(1)
    x = np.array([_bf16(v) for v in (rng.integers(-64, 64, size=H) / 8.0)], np.uint16)
    perm = rng.permutation(H)[:E]
    cs = [0.5, -1.0, 2.0, 0.25, 1.5, -0.75, 3.0, 1.0]
    W = np.zeros((E, H), np.uint16)
    for e in range(E):
        W[e, perm[e]] = _bf16(cs[e])
    logits = ref.router_logits(x, W)
    assert (logits == np.array([cs[e] * _f64(x[perm[e]]) for e in range(E)])).all()


def _brute_topk(logits, K):
    order = sorted(range(len(logits)), key=lambda e: (-logits[e], e))
    return order[:K]


def _softmax_closed(logits):
    m = max(logits)
    ex = [math.exp(v - m) for v in logits]
    z = math.fsum(ex)
    return [v / z for v in ex]


@pytest.mark.parametrize("E,K", [(8, 2), (512, 4), (64, 8)])
def test_topk_matches_brute_force_sort(ref, E, K):
    rng = np.random.default_rng(E + K)
    for trial in range(20):
        logits = rng.normal(scale=1.28, size=E)
        if trial % 3 == 0:  # exact ties must go to the lower index
            logits[rng.integers(E)] = logits.max()
            logits[rng.integers(E)] = logits.max()
        idx, w = ref.topk(logits, K)
        assert list(idx) == _brute_topk(list(logits), K)
        p = _softmax_closed(list(logits))
        assert np.allclose(w, [p[i] for i in idx], rtol=1e-12)
        idx_r, w_r = ref.topk(logits, K, renorm=True)
        assert list(idx_r) == list(idx)
        assert np.allclose(w_r, np.array([p[i] for i in idx]) / math.fsum(p[i] for i in idx), rtol=1e-12)


def test_topk_ties_prefer_lower_index(ref):
    logits = np.array([1.0, 3.0, 3.0, 0.5, 3.0, 2.0])
    idx, _ = ref.topk(logits, 4)
    assert list(idx) == [1, 2, 4, 5]


def test_topk_forced_indices(ref):
    logits = np.array([0.1, 0.4, -0.3, 2.0, 1.0])
    idx, w = ref.topk(logits, 2, forced=np.array([2, 0], np.int32))
    p = _softmax_closed(list(logits))
    assert list(idx) == [2, 0] and np.allclose(w, [p[2], p[0]], rtol=1e-14)
    with pytest.raises(ValueError):
        ref.topk(logits, 2, forced=np.array([5, 0], np.int32))


def test_softmax_two_expert_closed_form(ref):
    for a, b in ((0.0, 0.0), (1.0, -2.0), (30.0, 29.5), (-5.0, 3.0)):
        p = ref.softmax(np.array([a, b]))
        assert abs(p[0] - 1.0 / (1.0 + math.exp(b - a))) < 1e-15
        assert abs(p.sum() - 1.0) < 1e-15


# ---- SwiGLU -----------------------------------------------------------------

def test_silu_closed_forms(ref):
    e = math.e
    assert ref.silu(0.0) == 0.0
    assert abs(ref.silu(1.0) - e / (e + 1.0)) < 1e-15
    assert abs(ref.silu(-1.0) - (-1.0 / (e + 1.0))) < 1e-15
    assert abs(ref.silu(2.0) - 2.0 * e * e / (e * e + 1.0)) < 1e-15
    for z in (-7.5, -0.3, 0.7, 4.0, 12.0):  # z*sigmoid(z) == z*(1+tanh(z/2))/2
        assert abs(ref.silu(z) - z * (1.0 + math.tanh(z / 2.0)) / 2.0) < 1e-14 * max(1.0, abs(z))
    assert abs(ref.silu(40.0) - 40.0) < 1e-12 and abs(ref.silu(-40.0)) < 1e-15


def test_swiglu_gate_is_the_silu_operand(ref):
    h = ref.swiglu(np.array([1.0, 2.0]), np.array([2.0, 1.0]))
    e = math.e
    assert abs(h[0] - 2.0 * e / (e + 1.0)) < 1e-15      # silu(g=1) * u=2
    assert abs(h[1] - 2.0 * e * e / (e * e + 1.0)) < 1e-15


# ---- expert FFN --------------------------------------------------------------

def test_expert_ffn_constant_closed_form(ref):
    """Constant codes/scales per matrix: g_i = (cg*s+b)*sum(x), u_i =
    (cu*s+b)*sum(x), h_i = silu(g)*u, y = (cd*s+b)*I*h. Distinct gate and up
    constants catch a swap of the two."""
    H, I, G = 128, 64, 32
    rng = np.random.default_rng(2)
    x = rng.normal(size=H) / 8.0
    s, b = 0.0078125, 0.015625

    def mat(rows, cols, c, bb):
        return (np.full((rows, cols), c, np.uint8), np.full((rows, cols // G), _bf16(s), np.uint16),
                np.full((rows, cols // G), _bf16(bb), np.uint16))

    gate, up, down = mat(I, H, 3, b), mat(I, H, 11, -b), mat(H, I, 6, b)
    y = ref.expert_ffn(H, I, G, gate, up, down, x)
    sx = math.fsum(x)
    g = (3 * s + b) * sx
    u = (11 * s - b) * sx
    hval = g * (1.0 + math.tanh(g / 2.0)) / 2.0 * u
    expect = (6 * s + b) * I * hval
    assert np.allclose(y, expect, rtol=1e-12)


# ---- combine, gate, norm ----------------------------------------------------

def test_combine_one_hot_weight_selects_expert(ref):
    rng = np.random.default_rng(4)
    K, H = 4, 32
    y = rng.normal(size=(K + 1, H))
    for k in range(K):
        w = np.zeros(K)
        w[k] = 1.0
        assert (ref.combine(y, w, 0.0, np.zeros(H)) == y[k]).all()
    assert (ref.combine(y, np.zeros(K), 1.0, np.zeros(H)) == y[K]).all()
    r = rng.normal(size=H)
    assert (ref.combine(np.zeros((K + 1, H)), np.ones(K), 1.0, r) == r).all()


def test_shared_gate_is_sigmoid(ref):
    H = 16
    x = np.array([_bf16(1.0)] * H, np.uint16)
    assert ref.shared_gate(np.zeros(H, np.uint16), x) == 0.5
    wsg = np.zeros(H, np.uint16)
    wsg[3] = _bf16(2.0)
    assert abs(ref.shared_gate(wsg, x) - 1.0 / (1.0 + math.exp(-2.0))) < 1e-15


def test_rmsnorm_closed_forms(ref):
    out = ref.rmsnorm(np.array([3.0, 4.0]), 0.0)
    assert np.allclose(out, [3.0 / math.sqrt(12.5), 4.0 / math.sqrt(12.5)], rtol=1e-15)
    c, eps = -0.5, 1e-6
    out = ref.rmsnorm(np.full(64, c), eps)
    assert np.allclose(out, c / math.sqrt(c * c + eps), rtol=1e-15)
    xb = ref.rmsnorm_bf16(np.array([3.0, -4.0, 0.0, 5.0]), 0.0)
    # rms = sqrt(50/4); 3/3.5355 = 0.8485 -> bf16 0x3F59, etc.
    assert [int(v) for v in xb] == [int(ref.f64_to_bf16(v)[0]) for v in (3 / math.sqrt(12.5), -4 / math.sqrt(12.5),
                                                                          0.0, 5 / math.sqrt(12.5))]
    assert int(xb[2]) == 0 and int(xb[1]) & 0x8000


def test_rmsnorm_weighted_closed_forms(ref):
    """The standalone RMS norm with a weight vector: unit weight (None, or all
    ones) is the unweighted norm; [3, 4] with weights [0.5, 2] and a power of
    two weight follow by hand."""
    rng = np.random.default_rng(6)
    v = rng.normal(size=96)
    unit = ref.rmsnorm_bf16(v, 1e-6)
    assert (ref.rmsnorm_weighted_bf16(v, None, 1e-6) == unit).all()
    assert (ref.rmsnorm_weighted_bf16(v, np.full(96, _bf16(1.0), np.uint16), 1e-6) == unit).all()
    # a power-of-two weight scales exactly: the bf16 pattern moves by its exponent
    got = ref.rmsnorm_weighted_bf16(v, np.full(96, _bf16(4.0), np.uint16), 1e-6)
    assert (got.astype(np.int32) - unit.astype(np.int32) == np.where(unit & 0x7FFF, 2 << 7, 0)).all()
    w = np.array([_bf16(0.5), _bf16(2.0)], np.uint16)
    got = ref.rmsnorm_weighted_bf16(np.array([3.0, 4.0]), w, 0.0)
    rms = math.sqrt(12.5)
    assert [int(b) for b in got] == [_rne_bf16_bits(3.0 / rms * 0.5), _rne_bf16_bits(4.0 / rms * 2.0)]
    # a weight of -1 flips only the sign bit
    neg = ref.rmsnorm_weighted_bf16(v, np.full(96, _bf16(-1.0), np.uint16), 1e-6)
    assert (neg == (unit ^ 0x8000)).all()


# ---- the whole-layer glue (oracle/layer.py::layer_token) ---------------------

def _rne_bf16_bits(v: float) -> int:
    """bf16 bits nearest to v, ties to even, written from the format's
    definition (8 significant bits) with Python integers, not the oracle."""
    if v == 0.0:
        return 0x8000 if math.copysign(1.0, v) < 0 else 0
    m, e = math.frexp(abs(v))          # |v| = m * 2^e, 0.5 <= m < 1
    q = round(m * 256)                  # round() on a float is ties-to-even
    if q == 256:
        q, e = 128, e + 1
    f32 = np.float32(math.ldexp(q, e - 8)).view(np.uint32)
    return int((f32 >> 16) | (0x8000 if v < 0 else 0))


def _closed_form_layer(gate_w_on: bool, resid, forced, renorm, eps):
    """A layer whose every expert has constant codes per matrix and whose
    router rows are scaled one-hot vectors: logits, picks, expert outputs,
    combine and RMSNorm follow by hand (Python floats)."""
    H, I, G, E, K = 128, 64, 32, 6, 2
    s, b = 0.0078125, 0.015625
    xv = [1.0] * E + [((j * 7) % 11 - 5) / 8.0 for j in range(E, H)]
    x_bits = np.array([_bf16(v) for v in xv], np.uint16)
    alpha = [0.5, 2.0, -1.0, 1.5, 0.25, 3.0]          # logit of expert e = alpha_e * x_e = alpha_e
    router = np.zeros((E, H), np.uint16)
    for e in range(E):
        router[e, e] = _bf16(alpha[e])
    consts = {e: (1 + e, 14 - 2 * e, 3 + e) for e in range(E)}  # (gate, up, down) code per expert
    consts[E] = (9, 5, 12)                                      # the shared expert

    def mat(rows, cols, c, bb):
        return (np.full((rows, cols), c, np.uint8), np.full((rows, cols // G), _bf16(s), np.uint16),
                np.full((rows, cols // G), _bf16(bb), np.uint16))

    def weights(e):
        cg, cu, cd = consts[e]
        return mat(I, H, cg, b), mat(I, H, cu, -b), mat(H, I, cd, b)

    def y_const(e):
        cg, cu, cd = consts[e]
        sx = math.fsum(xv)
        g, u = (cg * s + b) * sx, (cu * s - b) * sx
        return (cd * s + b) * I * (g / (1.0 + math.exp(-g))) * u

    wsg = None
    gamma = 1.0
    if gate_w_on:
        wsg = np.zeros(H, np.uint16)
        wsg[0] = _bf16(0.5)
        gamma = 1.0 / (1.0 + math.exp(-0.5 * xv[0]))
    z = math.fsum(math.exp(a) for a in alpha)
    p = [math.exp(a) / z for a in alpha]
    idx = list(forced) if forced is not None else sorted(range(E), key=lambda e: (-alpha[e], e))[:K]
    w = [p[e] for e in idx]
    if renorm:
        t = sum(w)
        w = [v / t for v in w]
    r = list(xv) if resid is None else list(resid)
    out = [r[i] + sum(w[k] * y_const(idx[k]) for k in range(K)) + gamma * y_const(E) for i in range(H)]
    inv = 1.0 / math.sqrt(math.fsum(v * v for v in out) / H + eps)
    xn = [_rne_bf16_bits(v * inv) for v in out]
    ys = [y_const(e) for e in idx] + [y_const(E)]
    args = (H, I, E, K, G, x_bits, router, weights, weights(E))
    expect = dict(logits=alpha, idx=idx, w=w, y=ys, gamma=gamma, out=out, xn=xn)
    return args, wsg, expect


@pytest.mark.parametrize("gate_w_on,with_resid,forced,renorm,eps", [(False, False, None, False, 1e-6),
                                                                    (True, True, None, True, 0.25),
                                                                    (False, True, [2, 4], False, 1e-6),
                                                                    (True, False, [0, 5], True, 0.5)])
def test_layer_token_closed_form(ref, gate_w_on, with_resid, forced, renorm, eps):
    """oracle/layer.py::layer_token against a layer computed by hand: the
    residual default (r = widened x), the slot order (routed picks in rank
    order, the shared expert in row K), the shared-expert gate, forced picks,
    renormalisation and the RMSNorm hand-off to bf16 (an eps of the order of
    the mean square makes eps itself visible in the bf16 result)."""
    from oracle import layer as ref_layer
    resid = [0.25 * ((i % 9) - 4) for i in range(128)] if with_resid else None
    args, wsg, ex = _closed_form_layer(gate_w_on, resid, forced, renorm, eps)
    got = ref_layer.layer_token(*args, renorm=renorm, forced=forced,
                                resid=None if resid is None else np.array(resid), shared_gate_w=wsg, eps=eps)
    assert np.allclose(got["logits"], ex["logits"], rtol=0, atol=0)
    assert [int(v) for v in got["idx"]] == ex["idx"]
    assert np.allclose(got["w"], ex["w"], rtol=1e-13, atol=0)
    assert abs(got["gamma"] - ex["gamma"]) < 1e-15
    H = len(ex["out"])
    for k, v in enumerate(ex["y"]):
        assert np.allclose(got["y"][k], np.full(H, v), rtol=1e-12, atol=0), k
    assert np.allclose(got["out"], ex["out"], rtol=1e-12, atol=1e-15)
    assert [int(v) for v in got["xn"]] == ex["xn"]
