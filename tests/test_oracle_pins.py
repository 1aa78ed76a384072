"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each pin is written so that a plausible slip anywhere in the oracle (a swapped
nibble order, a dropped -8 offset, a wrong sign, a transposed operand, an
off-by-one in the rolling window, a wrong GQA mapping) fails at least one of
them; ``test_planted_mistakes_are_caught`` plants such slips into copies of the
oracle's functions and checks that the pins notice.
"""
import math
import os

import numpy as np
import pytest

from oracle import ref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------- fixtures
def load_handbuilt():
    cases, cur = [], None
    with open(os.path.join(GOLDEN, "q4_handbuilt_blocks.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, _, rest = line.partition(" ")
            if key == "case":
                cur = {"name": rest}
                cases.append(cur)
            elif key == "d":
                cur["d"] = int(rest, 16)
            elif key == "qs":
                cur["qs"] = np.array([int(b, 16) for b in rest.split()], np.uint8)
            elif key == "w":
                cur["w"] = np.array([float.fromhex(v) if v.lstrip("-").startswith("0x") else float(v)
                                     for v in rest.split()])
    return cases


HANDBUILT = load_handbuilt()


def same_bits_or_nan(a, b):
    """Equal as IEEE values including the sign of zero; NaN matches NaN."""
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    both_nan = np.isnan(a) & np.isnan(b)
    eq = (a == b) & (np.signbit(a) == np.signbit(b))
    return bool(np.all(both_nan | eq))


# ------------------------------------------------------------ pin functions
def pin_handbuilt(decode):
    """decode(qs[1,1,16], d[1,1]) -> 32 weights; must equal the hand-worked values."""
    for c in HANDBUILT:
        w = decode(c["qs"].reshape(1, 1, 16), np.array([[c["d"]]], np.uint16)).reshape(-1)
        assert same_bits_or_nan(w, c["w"]), c["name"]


def pin_single_block_dot(matvec):
    """K = 32: y = d * sum_j (q_j - 8) x_j, worked by hand for the ramp block."""
    qs = np.array([0xF0, 0xE1, 0xD2, 0xC3, 0xB4, 0xA5, 0x96, 0x87,
                   0x78, 0x69, 0x5A, 0x4B, 0x3C, 0x2D, 0x1E, 0x0F], np.uint8).reshape(1, 1, 16)
    d = np.array([[0x4000]], np.uint16)                  # d = 2
    x = np.zeros((1, 32), np.float32)
    x[0, 0] = 1.0                                        # w_0 = -8*2 = -16
    x[0, 15] = 0.5                                       # w_15 = 7*2 = 14 -> 7
    x[0, 16] = -1.0                                      # w_16 = 7*2 = 14 -> -14
    x[0, 31] = 0.25                                      # w_31 = -8*2 = -16 -> -4
    y = np.asarray(matvec(qs, d, x)).reshape(-1)
    assert y[0] == -16.0 + 7.0 - 14.0 - 4.0


def pin_one_hot_columns(matvec, qs, d):
    """One-hot x picks column j of the exactly dequantised W."""
    n, nb, _ = qs.shape
    k = nb * 32
    W = np.stack([HAND_ROW(qs[r], d[r]) for r in range(n)])
    for j in (0, 5, 15, 16, 31, 32, k - 1):
        x = np.zeros((1, k), np.float32)
        x[0, j] = 1.0
        y = np.asarray(matvec(qs, d, x)).reshape(-1)
        assert np.array_equal(y, W[:, j]), j


def HAND_ROW(qs_row, d_row):
    """Straight-line decode of one row, scalar Python, for the one-hot pin."""
    out = []
    for b in range(qs_row.shape[0]):
        scale = float(np.array([d_row[b]], np.uint16).view(np.float16)[0])
        for j in range(32):
            byte = int(qs_row[b][j % 16])
            q = (byte & 15) if j < 16 else (byte >> 4)
            out.append((q - 8) * scale)
    return np.array(out)


def pin_integer_matrix(matvec):
    """With d = 1 every weight is the integer q - 8, and with integer x the fp64
    product is exact: compare with numpy's int64 matmul."""
    rng = np.random.default_rng(7)
    n, k = 19, 96
    qs = rng.integers(0, 256, (n, k // 32, 16), dtype=np.uint8)
    d = np.full((n, k // 32), 0x3C00, np.uint16)
    x = rng.integers(-50, 51, (3, k)).astype(np.float32)
    codes = np.concatenate([qs & 15, qs >> 4], axis=-1).astype(np.int64).reshape(n, k) - 8
    want = x.astype(np.int64) @ codes.T
    got = np.asarray(matvec(qs, d, x))
    assert np.array_equal(got, want.astype(np.float64))


def pin_attention_list_model(attn, configs):
    """Brute force: simulate the rolling window as a plain list of the last W
    (k, v) pairs in arrival order, attend in pure Python, compare."""
    for (n_q, n_kv, hd, W) in configs:
        rng = np.random.default_rng([n_q, n_kv, hd, W])
        group = n_q // n_kv
        k_cache = np.zeros((n_kv, W, hd), np.uint16)
        v_cache = np.zeros((n_kv, W, hd), np.uint16)
        history = []                                      # list of (k, v) fp32 [n_kv, hd]
        for P in range(3 * W + 1):
            k_new = rng.standard_normal((n_kv, hd)).astype(np.float32)
            v_new = rng.standard_normal((n_kv, hd)).astype(np.float32)
            ref.c_kv_append(k_cache, v_cache, k_new, v_new, P)
            history.append((ref.bf16_to_f64(ref.f32_to_bf16(k_new)), ref.bf16_to_f64(ref.f32_to_bf16(v_new))))
            window = history[-W:]
            q = rng.standard_normal((n_q, hd)).astype(np.float32)
            got = attn(q, k_cache, v_cache, P)
            for h in range(n_q):
                kvh = h // group
                s = [sum(float(q[h, c]) * kv[0][kvh, c] for c in range(hd)) / math.sqrt(hd) for kv in window]
                m = max(s)
                e = [math.exp(v - m) for v in s]
                tot = sum(e)
                want = [sum(e[j] * window[j][1][kvh, c] for j in range(len(window))) / tot for c in range(hd)]
                np.testing.assert_allclose(got[h], want, rtol=1e-12, atol=1e-12)


# ------------------------------------------- error metric and composed pins
def pin_gemv_error(metric):
    """The normalised GEMV error, worked by hand.  x = (3, 4) has norm 5; the
    rows w0 = (3, 4) and w1 = (0, 2) have norms 5 and 2 (their columns have
    norms 3 and sqrt(20), so a row/column slip changes the value)."""
    x = np.array([[3.0, 4.0]])
    W = np.array([[3.0, 4.0], [0.0, 2.0]])
    y_ref = np.array([[25.0, 8.0]])
    # errors 0.5 on both outputs: 0.5 / (5 * 5) = 0.02 and 0.5 / (5 * 2) = 0.05
    assert metric(y_ref + 0.5, y_ref, x, W) == 0.05
    # a second activation row (0, 1), norm 1: an error of -0.3 on output 1
    # gives 0.3 / (1 * 2) = 0.15, larger than row 0's 0.05
    x2 = np.array([[3.0, 4.0], [0.0, 1.0]])
    y2_ref = np.array([[25.0, 8.0], [4.0, 2.0]])
    y2 = y2_ref + np.array([[0.5, 0.5], [0.0, -0.3]])
    assert metric(y2, y2_ref, x2, W) == pytest.approx(0.15, rel=1e-15)
    assert metric(y2_ref, y2_ref, x2, W) == 0.0


def pin_attn_error(metric):
    """The normalised attention error, worked by hand: two kv heads of two
    valid slots and head_dim 2, group 1.  Head 0: p = (0.6, 0.8) (norm 1),
    V = [[3, 1], [4, 0]] (columns of norms 5 and 1).  Head 1: p = (1, 0),
    V = [[0, 2], [0, 0]] (column norms 0 and 2)."""
    probs = np.array([[0.6, 0.8], [1.0, 0.0]])
    Vv = np.array([[[3.0, 1.0], [4.0, 0.0]], [[0.0, 2.0], [0.0, 0.0]]])
    o_ref = np.array([[5.0, 0.6], [0.0, 2.0]])
    # head 0 errors (0.5, 0.1): 0.5/5 = 0.1, 0.1/1 = 0.1; head 1 error 0.5 on dim 1: 0.5/2 = 0.25
    o = o_ref + np.array([[0.5, 0.1], [0.0, 0.5]])
    assert metric(o, o_ref, probs, Vv, 1) == 0.25
    o = o_ref + np.array([[0.5, -0.3], [0.0, 0.0]])
    assert metric(o, o_ref, probs, Vv, 1) == pytest.approx(0.3, rel=1e-15)
    # group 2: both query heads read kv head 0
    o2_ref = np.array([[5.0, 0.6], [5.0, 0.6]])
    o2 = o2_ref + np.array([[0.0, 0.0], [1.0, 0.0]])
    assert metric(o2, o2_ref, np.array([[0.6, 0.8], [0.6, 0.8]]), Vv, 2) == pytest.approx(0.2, rel=1e-15)


def pin_attn_probs(probs):
    """Softmax probabilities of hand-built keys: with scale 1/2, q = (2, 0) and
    keys (1, 0), (0, 1) the scores are 1 and 0, so p = (e, 1) / (1 + e); one
    valid key gives p = 1; the second kv head (keys (0, 1), (1, 0)) swaps them."""
    one, zero = 0x3F80, 0x0000                      # bf16 1.0 and 0.0
    kc = np.array([[[one, zero], [zero, one], [one, one]],
                   [[zero, one], [one, zero], [one, one]]], np.uint16)   # n_kv 2, W 3, hd 2
    q = np.array([[2.0, 0.0], [2.0, 0.0]], np.float32)
    e = math.e
    P = probs(q, kc, 1, 0.5)                         # positions 0 and 1 written
    np.testing.assert_allclose(P, [[e / (1 + e), 1 / (1 + e)], [1 / (1 + e), e / (1 + e)]], rtol=1e-15)
    assert np.array_equal(probs(q, kc, 0, 0.5), np.ones((2, 1)))
    # wrapped (pos 7 >= W): all three slots, scores (1, 0, 1) and (0, 1, 1)
    P = probs(q, kc, 7, 0.5)
    np.testing.assert_allclose(P[0], np.array([e, 1.0, e]) / (2 * e + 1), rtol=1e-15)
    np.testing.assert_allclose(P[1], np.array([1.0, e, e]) / (2 * e + 1), rtol=1e-15)


def _bf16_round(v):
    """bf16 (nearest-even) of float32 values by torch's CPU cast, widened back."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(np.asarray(v, np.float32))).to(torch.bfloat16)
    return t.to(torch.float64).numpy()


def pin_decoder_layer(layer):
    """Closed forms of one decoder layer (dim 4, 4 query / 2 kv heads of
    head_dim 1, FFN 4, window 3) in special cases:
    (a) Wo = W2 = 0: out = h = x exactly, at any position;
    (b) position 0 (one valid key): o of query head h is the stored (bf16)
        v of kv head h // 2;
    (c) Wo = I, W2 = 0 at position 0: out = x + o, the residual is x;
    (d) Wq = Wk = 0, Wv picks column 0, Wo = I, W1 = 2I, W3 = 3I, W2 = I:
        out_i = h_i + silu(2 n2_i) * 3 n2_i with n2 = RMSNorm(h), h = x + o."""
    rng = np.random.default_rng(21)
    D, nq, nkv, W = 4, 4, 2, 3
    eps = ref.RMS_EPS
    x = np.array([1.5, -0.5, 2.0, -1.0])
    Z = np.zeros((D, D))
    I = np.eye(D)

    def weights(**kw):
        w = {"wq": rng.standard_normal((nq, D)), "wk": rng.standard_normal((nkv, D)),
             "wv": rng.standard_normal((nkv, D)), "wo": rng.standard_normal((D, nq)),
             "w1": rng.standard_normal((D, D)), "w3": rng.standard_normal((D, D)),
             "w2": rng.standard_normal((D, D))}
        w.update(kw)
        return w

    def caches():
        return (synth_bf16((nkv, W, 1), 1), synth_bf16((nkv, W, 1), 2))

    # (a)
    for pos in (0, 1, 5):
        kc, vc = caches()
        st = layer(x, weights(wo=np.zeros((D, nq)), w2=Z), kc, vc, pos, nq, nkv)
        assert np.array_equal(st["out"], x) and np.array_equal(st["h"], x)
    # (b) and (c)
    kc, vc = caches()
    w = weights(wo=np.eye(D, nq), w2=Z)
    st = layer(x, w, kc, vc, 0, nq, nkv)
    n = x / math.sqrt(float(np.mean(x * x)) + eps)
    v_stored = _bf16_round(w["wv"] @ n)
    assert np.array_equal(st["o"], v_stored[[0, 0, 1, 1]])
    assert np.array_equal(st["out"], x + v_stored[[0, 0, 1, 1]])
    # (d)
    kc, vc = caches()
    wv = np.zeros((nkv, D)); wv[:, 0] = 1.0
    st = layer(x, weights(wq=np.zeros((nq, D)), wk=np.zeros((nkv, D)), wv=wv, wo=np.eye(D, nq),
                          w1=2 * I, w3=3 * I, w2=I), kc, vc, 0, nq, nkv)
    o = float(_bf16_round([x[0] / math.sqrt(float(np.mean(x * x)) + eps)])[0])
    h = x + o
    r = 1.0 / math.sqrt(sum(v * v for v in h) / D + eps)
    want = [hi + (2 * hi * r) / (1 + math.exp(-2 * hi * r)) * 3 * hi * r for hi in h]
    np.testing.assert_allclose(st["out"], want, rtol=1e-14)


def synth_bf16(shape, tid):
    import synth

    return synth.bf16_normal(shape, 0, tid)


def pin_encoder_layer(layer):
    """Closed forms of one encoder layer (3 rows, dim 2, 2 heads of head_dim 1,
    FFN 2, 2 history rows):
    (a) Wo = Wdown = 0: out = X exactly;
    (b) window 1 (a row sees only itself), Wqkv = [0; 0; I] (v = RMSNorm(X)),
        Wo = I, Wdown = 0: out = X + RMSNorm(X);
    (c) Wo = 0, Wup = 1.5 I, Wdown = 2 I: out = X + 2 gelu(1.5 RMSNorm(X))."""
    rng = np.random.default_rng(22)
    X = np.array([[1.0, -2.0], [0.5, 0.25], [-3.0, 1.0]])
    D, eps = 2, ref.RMS_EPS
    kh, vh = rng.standard_normal((2, D)), rng.standard_normal((2, D))
    Z = np.zeros((D, D))

    def weights(**kw):
        w = {"wqkv": rng.standard_normal((3 * D, D)), "wo": rng.standard_normal((D, D)),
             "wup": rng.standard_normal((D, D)), "wdown": rng.standard_normal((D, D))}
        w.update(kw)
        return w

    n = np.array([[v / math.sqrt((row[0] ** 2 + row[1] ** 2) / D + eps) for v in row] for row in X])
    assert np.array_equal(layer(X, weights(wo=Z, wdown=Z), kh, vh, 3, 2, 1), X)
    wqkv = np.zeros((3 * D, D)); wqkv[2 * D:] = np.eye(D)
    out = layer(X, weights(wqkv=wqkv, wo=np.eye(D), wdown=Z), kh, vh, 1, 2, 1)
    np.testing.assert_allclose(out, X + n, rtol=1e-14)
    out = layer(X, weights(wo=Z, wup=1.5 * np.eye(D), wdown=2 * np.eye(D)), kh, vh, 3, 2, 1)
    g = np.array([[1.5 * v * (1 + math.erf(1.5 * v / math.sqrt(2))) for v in row] for row in n])
    np.testing.assert_allclose(out, X + g, rtol=1e-14)


# ------------------------------------------------------------------- tests
def test_half_decode_all_patterns(oracle_c):
    """The C oracle's hand-written fp16 decode equals numpy's cast on all 65536 patterns."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    want = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle_c.vr_half_to_double(int(b)) for b in bits])
    assert same_bits_or_nan(got, want)


def test_bf16_rounding_matches_torch(oracle_c):
    """Both oracle bf16 roundings equal torch's CPU cast (RNE) away from NaN."""
    import torch

    rng = np.random.default_rng(1)
    f = np.concatenate([
        rng.standard_normal(20000).astype(np.float32),
        (rng.standard_normal(2000) * 1e-39).astype(np.float32),     # subnormals
        np.array([0.0, -0.0, np.inf, -np.inf, 3.4028235e38, -3.4028235e38, 1.0 + 2**-8,
                  1.0 + 3 * 2**-8], np.float32),
        # exact ties at every exponent: a kept part plus 0x8000 in the dropped bits
        (rng.integers(0, 0x7F7F, 2000, dtype=np.uint32) << 16 | 0x8000).astype(np.uint32).view(np.float32),
    ])
    want = torch.from_numpy(f.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got_np = ref.f32_to_bf16(f)
    got_c = np.array([oracle_c.vr_f32_to_bf16(float(v)) for v in f], np.uint16)
    assert np.array_equal(got_np, want)
    assert np.array_equal(got_c, want)
    assert oracle_c.vr_f32_to_bf16(float("nan")) == 0x7FC0
    assert ref.f32_to_bf16(np.array([np.nan], np.float32))[0] == 0x7FC0


def test_handbuilt_blocks_c_and_numpy():
    pin_handbuilt(lambda qs, d: ref.c_dequant_f32(qs, d))
    pin_handbuilt(lambda qs, d: ref.dequant_f32(qs, d))


def test_bf16_dequant_ties():
    rows = []
    with open(os.path.join(GOLDEN, "bf16_ties.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                a, b = line.split()
                rows.append((int(a, 16), int(b, 16)))
    qs = np.full((len(rows), 1, 16), 0x99, np.uint8)       # every code 9 -> q - 8 = 1
    d = np.array([[a] for a, _ in rows], np.uint16)
    want = np.array([b for _, b in rows], np.uint16)
    assert np.all(ref.c_dequant_bf16(qs, d) == want[:, None])
    assert np.all(ref.dequant_bf16(qs, d) == want[:, None])


def test_dequant_fp32_is_exact():
    """(q-8)*d is exactly representable in fp32 for every fp16 d: the fp32
    output widened back to float64 equals the float64 product."""
    rng = np.random.default_rng(3)
    qs = rng.integers(0, 256, (64, 8, 16), dtype=np.uint8)
    d = rng.integers(0, 0x7C00, (64, 8), dtype=np.uint16)   # all finite non-negative fp16
    d[::2] |= 0x8000
    exact = ref.q4_weights(qs, d)
    assert np.array_equal(ref.c_dequant_f32(qs, d).astype(np.float64), exact)


def test_matvec_single_block_by_hand():
    pin_single_block_dot(ref.c_matvec)
    pin_single_block_dot(ref.matvec)
    pin_single_block_dot(ref.c_matvec_blocksum)


def test_matvec_one_hot_columns():
    rng = np.random.default_rng(11)
    qs = rng.integers(0, 256, (9, 3, 16), dtype=np.uint8)
    d = (np.abs(rng.standard_normal((9, 3))) * 0.5).astype(np.float16).view(np.uint16)
    pin_one_hot_columns(ref.c_matvec, qs, d)
    pin_one_hot_columns(ref.matvec, qs, d)


def test_matvec_zero_codes():
    qs = np.full((5, 4, 16), 0x88, np.uint8)
    d = np.full((5, 4), 0x3C00, np.uint16)
    x = np.ones((2, 128), np.float32)
    assert np.all(ref.c_matvec(qs, d, x) == 0.0)


def test_matvec_integer_exact():
    pin_integer_matrix(ref.c_matvec)
    pin_integer_matrix(ref.matvec)
    pin_integer_matrix(ref.c_matvec_blocksum)


def test_matvec_routes_agree():
    """Dense route (dequantise then fp64 matmul) == block-sum identity == numpy twin."""
    import synth

    qs, d = synth.q4_blocks(300, 3072, 0, 12345)
    x = synth.activations(3, 3072, 0, 54321)
    y_dense = ref.c_matvec(qs, d, x)
    y_block = ref.c_matvec_blocksum(qs, d, x)
    y_np = ref.matvec(qs, d, x)
    scale = np.abs(y_dense).max()
    assert np.max(np.abs(y_dense - y_block)) <= 1e-12 * scale
    assert np.max(np.abs(y_dense - y_np)) <= 1e-12 * scale
    # row sampling of the C oracle returns the same rows
    y_rows = ref.c_matvec(qs, d, x, row0=17, nrows=40)
    assert np.array_equal(y_rows, y_dense[:, 17:57])


def test_rolling_slots_bruteforce():
    """slot = pos mod W: after appending 0..P the slots hold exactly the last
    min(P+1, W) positions, each once (list model)."""
    for W in (1, 2, 3, 5, 8192):
        slots = {}
        last = []
        top = 3 * W + 5 if W < 100 else 2 * W + 300
        for P in range(top + 1):
            s = int(ref.c_lib().vr_kv_slot(P, W))
            assert s == ref.kv_slot(P, W)
            slots[s] = P
            last.append(P)
            last = last[-W:]
            assert sorted(slots.values()) == last
            assert len(slots) == ref.valid_slots(P, W)
            assert set(slots.keys()) == set(range(ref.valid_slots(P, W)))


def test_kv_append_c_equals_numpy():
    rng = np.random.default_rng(5)
    kc1 = np.zeros((3, 7, 16), np.uint16); vc1 = kc1.copy()
    kc2 = kc1.copy(); vc2 = kc1.copy()
    for P in range(20):
        k = rng.standard_normal((3, 16)).astype(np.float32)
        v = rng.standard_normal((3, 16)).astype(np.float32)
        ref.c_kv_append(kc1, vc1, k, v, P)
        ref.kv_append(kc2, vc2, k, v, P)
    assert np.array_equal(kc1, kc2) and np.array_equal(vc1, vc2)


TINY_ATTN = [(1, 1, 1, 1), (2, 1, 4, 3), (4, 2, 8, 5), (2, 2, 4, 1), (4, 1, 8, 3)]


def test_attention_bruteforce_c():
    pin_attention_list_model(lambda q, kc, vc, P: ref.c_gqa_attn(q, kc, vc, P), TINY_ATTN)


def test_attention_bruteforce_numpy():
    pin_attention_list_model(lambda q, kc, vc, P: ref.gqa_attn(q, kc, vc, P), TINY_ATTN)


def test_attention_invariants():
    import synth

    n_q, n_kv, hd, W = 8, 2, 16, 37
    kc = synth.bf16_normal((n_kv, W, hd), 0, 1)
    vc = synth.bf16_normal((n_kv, W, hd), 0, 2)
    q = synth.activations(n_q, hd, 0, 3)
    V = ref.bf16_to_f64(vc)
    # one valid key -> o = v exactly
    o = ref.c_gqa_attn(q, kc, vc, 0)
    for h in range(n_q):
        assert np.array_equal(o[h], V[h // 4, 0])
    # q = 0 -> mean of the valid V rows
    P = 20
    o = ref.c_gqa_attn(np.zeros_like(q), kc, vc, P)
    for h in range(n_q):
        np.testing.assert_allclose(o[h], V[h // 4, :P + 1].mean(axis=0), rtol=1e-12, atol=1e-13)
    # wrapped: permuting the slots leaves o unchanged (ring == compaction)
    P = 3 * W + 4
    perm = np.random.default_rng(0).permutation(W)
    o1 = ref.c_gqa_attn(q, kc, vc, P)
    o2 = ref.c_gqa_attn(q, np.ascontiguousarray(kc[:, perm]), np.ascontiguousarray(vc[:, perm]), P)
    np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-13)
    # group size 1 is plain multi-head attention: head h reads kv head h
    o_mha = ref.c_gqa_attn(q[:2], kc, vc, P)
    for h in range(2):
        o_single = ref.c_gqa_attn(q[h:h + 1], np.ascontiguousarray(kc[h:h + 1]), np.ascontiguousarray(vc[h:h + 1]), P)
        np.testing.assert_allclose(o_mha[h], o_single[0], rtol=1e-12, atol=1e-13)
    # split-KV combine with any split count equals the unsplit result
    for ns in (1, 2, 3, 7, W):
        np.testing.assert_allclose(ref.combine_partials(ref.split_partials(q, kc, vc, P, ns)), o1,
                                   rtol=1e-12, atol=1e-13)
    # C and numpy twins agree
    np.testing.assert_allclose(ref.gqa_attn(q, kc, vc, P), o1, rtol=1e-12, atol=1e-13)


def test_rmsnorm_silu_gelu_closed_forms():
    eps = ref.RMS_EPS
    for c in (0.1, 1.0, -3.0, 250.0):
        r = ref.rmsnorm(np.full(3072, c))
        np.testing.assert_allclose(r, np.sign(c) / np.sqrt(1 + eps / c ** 2), rtol=1e-14)
    assert ref.silu(0.0) == 0.0
    np.testing.assert_allclose(ref.silu(np.array([30.0, -30.0, 1.0])),
                               [30.0 - 30.0 * math.exp(-30.0) / (1 + math.exp(-30.0)),
                                -30.0 * math.exp(-30.0) / (1 + math.exp(-30.0)), 1 / (1 + math.exp(-1))],
                               rtol=1e-14)
    assert ref.gelu(0.0) == 0.0
    xs = np.array([-6.0, -1.0, -0.3, 0.5, 2.0, 9.0])
    want = [0.5 * v * (1 + math.erf(v / math.sqrt(2))) for v in xs]
    np.testing.assert_allclose(ref.gelu(xs), want, rtol=1e-14)
    assert abs(ref.gelu(40.0) - 40.0) < 1e-12


def test_error_metrics_by_hand():
    pin_gemv_error(ref.gemv_error)
    pin_attn_error(ref.attn_error)


def test_attention_probabilities_by_hand():
    pin_attn_probs(ref.attn_probs)


def test_bf16_widening_matches_torch():
    """bf16 -> float64 widening equals torch's bf16 -> fp32 cast on all 65536 patterns."""
    import torch

    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    want = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).to(torch.float32).numpy()
    with np.errstate(invalid="ignore"):               # NaN patterns widen to NaN
        assert same_bits_or_nan(ref.bf16_to_f64(bits), want.astype(np.float64))


def test_decoder_layer_closed_forms():
    pin_decoder_layer(ref.decoder_layer)


def test_encoder_layer_closed_forms():
    pin_encoder_layer(ref.encoder_layer)


def test_window_attention_bruteforce():
    """Encoder sliding window: query i (position q0+i) sees j with p-W < j <= p."""
    rng = np.random.default_rng(9)
    nh, hd, W, nhist, nq = 2, 3, 4, 5, 3
    Q = rng.standard_normal((nq, nh * hd))
    K = rng.standard_normal((nhist + nq, nh * hd))
    V = rng.standard_normal((nhist + nq, nh * hd))
    got = ref.window_attn(Q, K, V, nhist, W, nh, hd)
    for i in range(nq):
        p = nhist + i
        vis = [j for j in range(nhist + nq) if p - W < j <= p]
        assert len(vis) == W
        for h in range(nh):
            sl = slice(h * hd, (h + 1) * hd)
            s = [float(Q[i, sl] @ K[j, sl]) / math.sqrt(hd) for j in vis]
            e = [math.exp(v - max(s)) for v in s]
            want = sum(e[t] * V[vis[t], sl] for t in range(W)) / sum(e)
            np.testing.assert_allclose(got[i, sl], want, rtol=1e-12)


def pin_adapter(fn):
    """Closed forms of the adapter: with W1 = a [I | 0] (picking the first
    columns) and W2 = b I the output is b gelu(a x[:, :n]); W2 = 0 gives 0."""
    rng = np.random.default_rng(31)
    X = rng.standard_normal((3, 8))
    W1 = np.zeros((4, 8)); W1[:, :4] = 1.5 * np.eye(4)
    out = fn(X, W1, -2.0 * np.eye(4))
    want = [[-2.0 * 0.5 * 1.5 * v * (1 + math.erf(1.5 * v / math.sqrt(2))) for v in row[:4]] for row in X]
    np.testing.assert_allclose(out, want, rtol=1e-14)
    assert np.array_equal(fn(X, rng.standard_normal((4, 8)), np.zeros((4, 4))), np.zeros((3, 4)))


def test_adapter_closed_forms():
    pin_adapter(ref.adapter)

    def gelu_after_second(Xd, W1, W2):
        return ref.gelu(np.asarray(Xd) @ np.asarray(W1).T @ np.asarray(W2).T)

    def no_gelu(Xd, W1, W2):
        return np.asarray(Xd) @ np.asarray(W1).T @ np.asarray(W2).T

    for bad in (gelu_after_second, no_gelu):
        with pytest.raises(AssertionError):
            pin_adapter(bad)


def test_downsample_order():
    X = np.arange(8 * 3).reshape(8, 3)
    Y = ref.downsample_rows(X, 4)
    assert Y.shape == (2, 12)
    assert list(Y[1]) == list(range(12, 24))


def test_argmax_lowest_index():
    assert ref.argmax_lowest([1.0, 3.0, 3.0, 2.0]) == 1
    assert ref.argmax_lowest([-1.0, -1.0]) == 0


def test_shape_readings_match_page_footprints():
    """Parameter-count cross-check of the shape readings against the pages'
    footprints (tests/golden/footprint.txt): untied embedding + LM head and an
    ungated encoder FFN fit; the alternatives fit worse."""
    fp = {}
    with open(os.path.join(GOLDEN, "footprint.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                key, val, unit, tol = line.split()[:4]
                fp[key] = (float(val), unit, float(tol))
    dec_layer = 4096 * 3072 + 2 * 1024 * 3072 + 3072 * 4096 + 3 * 9216 * 3072
    assert dec_layer == 116_391_936
    enc_layer = 3 * 1280 * 1280 + 1280 * 1280 + 2 * 5120 * 1280
    vocab = int(fp["vocab"][0])
    embed = vocab * 3072
    adapter = 5120 * 3072 + 3072 * 3072
    total = 26 * dec_layer + 2 * embed + 32 * enc_layer + adapter
    assert total == 4_485_808_128

    def within(key, value):
        want, _, tol = fp[key]
        return abs(value - want) <= tol * want

    assert within("bf16_weights", total * 2 / 1e9)
    assert within("f16_gpu_cache", total * 2 / 2 ** 30)
    assert within("q4_gguf", total * 18 / 32 / 1e9)
    assert within("kv_cache_max", 26 * 8192 * 1024 * 2 * 4 / 1e9)
    assert within("embedding_f32", embed * 4 / 2 ** 30)
    gated = total + 32 * 5120 * 1280
    tied = total - embed
    assert abs(gated * 2 / 1e9 - 8.9) > abs(total * 2 / 1e9 - 8.9)
    assert abs(tied * 2 / 1e9 - 8.9) > abs(total * 2 / 1e9 - 8.9)


# ------------------------------------------------------- planted mistakes
def test_planted_mistakes_are_caught():
    """Copies of the oracle's functions with one plausible slip each must fail a pin."""
    def swapped_nibbles(qs, d):
        codes = np.concatenate([qs >> 4, qs & 0x0F], axis=-1).astype(np.int64)
        return ((codes - 8) * ref.half_to_f64(d)[:, :, None]).reshape(qs.shape[0], -1)

    def no_offset(qs, d):
        codes = np.concatenate([qs & 0x0F, qs >> 4], axis=-1).astype(np.int64)
        return (codes * ref.half_to_f64(d)[:, :, None]).reshape(qs.shape[0], -1)

    def interleaved_nibbles(qs, d):
        codes = np.stack([qs & 0x0F, qs >> 4], axis=-1).reshape(qs.shape[0], qs.shape[1], 32).astype(np.int64)
        return ((codes - 8) * ref.half_to_f64(d)[:, :, None]).reshape(qs.shape[0], -1)

    for bad in (swapped_nibbles, no_offset, interleaved_nibbles):
        with pytest.raises(AssertionError):
            pin_handbuilt(bad)

    def transposed_matvec(qs, d, x):
        W = ref.q4_weights(qs, d)
        x = np.atleast_2d(x).astype(np.float64)
        return (W[:, :x.shape[1]] @ x[:, :W.shape[0]].T).T if W.shape[0] == W.shape[1] else x @ W[:, ::-1].T

    with pytest.raises(AssertionError):
        pin_integer_matrix(transposed_matvec)

    def attn_off_by_one(q, kc, vc, P):           # drops the newest position
        return ref.gqa_attn(q, kc, vc, max(P - 1, 0))

    with pytest.raises(AssertionError):
        pin_attention_list_model(attn_off_by_one, [(2, 1, 4, 3)])

    def attn_wrong_group(q, kc, vc, P):          # interleaved head -> kv mapping
        n_kv = kc.shape[0]
        out = np.empty((q.shape[0], kc.shape[2]))
        for h in range(q.shape[0]):
            out[h] = ref.gqa_attn(q[h:h + 1], kc[h % n_kv:h % n_kv + 1], vc[h % n_kv:h % n_kv + 1], P)[0]
        return out

    with pytest.raises(AssertionError):
        pin_attention_list_model(attn_wrong_group, [(4, 2, 8, 5)])


def test_planted_mistakes_in_metric_and_layers_are_caught():
    """Slips in the error metric, the probabilities and the composed layers fail a pin."""
    def metric_column_norms(y, y_ref, x, w):         # norms of W's columns, not its rows
        return ref.gemv_error(y, y_ref, x, np.asarray(w).T)

    def metric_squared_x(y, y_ref, x, w):
        x = np.atleast_2d(np.asarray(x, np.float64))
        return ref.gemv_error(y, y_ref, x * np.linalg.norm(x, axis=1, keepdims=True), w)

    def metric_mean(y, y_ref, x, w):
        y, y_ref = np.atleast_2d(y), np.atleast_2d(y_ref)
        xn = np.linalg.norm(np.atleast_2d(x), axis=1)[:, None]
        wn = np.linalg.norm(w, axis=1)[None, :]
        return float(np.mean(np.abs(y - y_ref) / (xn * wn)))

    for bad in (metric_column_norms, metric_squared_x, metric_mean):
        with pytest.raises(AssertionError):
            pin_gemv_error(bad)

    def attn_metric_row_norms(o, o_ref, probs, Vv, group):   # norms over slots of a dim, swapped
        return ref.attn_error(o, o_ref, probs, np.swapaxes(Vv, 1, 2), group)

    def attn_metric_wrong_group(o, o_ref, probs, Vv, group):
        return ref.attn_error(o, o_ref, probs, Vv[::-1], group)

    for bad in (attn_metric_row_norms, attn_metric_wrong_group):
        with pytest.raises(AssertionError):
            pin_attn_error(bad)

    def probs_no_scale(q, kc, pos, scale=None):
        return ref.attn_probs(q, kc, pos, 1.0)

    def probs_sign(q, kc, pos, scale=None):
        return ref.attn_probs(-np.asarray(q), kc, pos, scale)

    def probs_drop_newest(q, kc, pos, scale=None):
        return ref.attn_probs(q, kc, max(pos - 1, 0), scale)

    for bad in (probs_no_scale, probs_sign, probs_drop_newest):
        with pytest.raises(AssertionError):
            pin_attn_probs(bad)

    def layer_residual_from_norm(x, Wd, kc, vc, pos, nq, nkv, eps=ref.RMS_EPS):
        st = ref.decoder_layer(x, Wd, kc, vc, pos, nq, nkv, eps)
        h = st["n"] + Wd["wo"] @ st["o"]
        st["h"] = h
        st["out"] = h + Wd["w2"] @ (ref.silu(Wd["w1"] @ ref.rmsnorm(h)) * (Wd["w3"] @ ref.rmsnorm(h)))
        return st

    def layer_ffn_from_first_norm(x, Wd, kc, vc, pos, nq, nkv, eps=ref.RMS_EPS):
        st = ref.decoder_layer(x, Wd, kc, vc, pos, nq, nkv, eps)
        st["out"] = st["h"] + Wd["w2"] @ (ref.silu(Wd["w1"] @ st["n"]) * (Wd["w3"] @ st["n"]))
        return st

    def layer_gate_on_up(x, Wd, kc, vc, pos, nq, nkv, eps=ref.RMS_EPS):
        st = ref.decoder_layer(x, Wd, kc, vc, pos, nq, nkv, eps)
        st["out"] = st["h"] + Wd["w2"] @ ((Wd["w1"] @ st["n2"]) * ref.silu(Wd["w3"] @ st["n2"]))
        return st

    def layer_interleaved_gqa(x, Wd, kc, vc, pos, nq, nkv, eps=ref.RMS_EPS):
        st = ref.decoder_layer(x, Wd, kc, vc, pos, nq, nkv, eps)
        hd = kc.shape[2]
        q = st["q"].reshape(nq, hd)
        o = np.stack([ref.gqa_attn(q[h:h + 1], kc[h % nkv:h % nkv + 1], vc[h % nkv:h % nkv + 1], pos)[0]
                      for h in range(nq)]).reshape(-1)
        st["o"] = o
        st["h"] = x + Wd["wo"] @ o
        n2 = ref.rmsnorm(st["h"])
        st["out"] = st["h"] + Wd["w2"] @ (ref.silu(Wd["w1"] @ n2) * (Wd["w3"] @ n2))
        return st

    for bad in (layer_residual_from_norm, layer_ffn_from_first_norm, layer_gate_on_up, layer_interleaved_gqa):
        with pytest.raises(AssertionError):
            pin_decoder_layer(bad)

    def enc_residual_from_norm(X, Wd, kh, vh, window, nh, hd, eps=ref.RMS_EPS):
        return ref.encoder_layer(X, Wd, kh, vh, window, nh, hd, eps) - np.asarray(X) + ref.rmsnorm(X)

    def enc_gelu_after_down(X, Wd, kh, vh, window, nh, hd, eps=ref.RMS_EPS):
        W2 = dict(Wd)
        W2["wdown"] = np.zeros_like(Wd["wdown"])
        h = ref.encoder_layer(X, W2, kh, vh, window, nh, hd, eps)
        return h + ref.gelu((ref.rmsnorm(h) @ Wd["wup"].T) @ Wd["wdown"].T)

    def enc_window_one_wider(X, Wd, kh, vh, window, nh, hd, eps=ref.RMS_EPS):
        return ref.encoder_layer(X, Wd, kh, vh, window + 1, nh, hd, eps)

    for bad in (enc_residual_from_norm, enc_gelu_after_down, enc_window_one_wider):
        with pytest.raises(AssertionError):
            pin_encoder_layer(bad)


# ------------------------------------------------------------ paged caches
def pin_paged(to_cache, append):
    """Brute force on a tiny pool whose every element holds a code of its own
    (page, head, row, col): the gathered cache and the appended slot must sit
    exactly where the page table says (reading R16), and appending through
    the pages must equal appending to the gathered cache."""
    P, n_kv, hd = 7, 2, 3
    pool = np.zeros((P, n_kv, ref.PAGE_SLOTS, hd), np.uint16)
    for p in range(P):
        for h in range(n_kv):
            for r in range(ref.PAGE_SLOTS):
                for c in range(hd):
                    pool[p, h, r, c] = ((p * n_kv + h) * ref.PAGE_SLOTS + r) * hd + c
    table = np.array([5, 0, 3], np.int32)                  # W = 192 slots in pages 5, 0, 3
    W = len(table) * ref.PAGE_SLOTS
    cache = to_cache(pool, table)
    assert cache.shape == (n_kv, W, hd)
    for h in range(n_kv):
        for slot in range(W):
            for c in range(hd):
                page, row = int(table[slot // ref.PAGE_SLOTS]), slot % ref.PAGE_SLOTS
                assert cache[h, slot, c] == ((page * n_kv + h) * ref.PAGE_SLOTS + row) * hd + c
    rng = np.random.default_rng(11)
    kp, vp = pool.copy(), pool.copy()
    kc, vc = to_cache(kp, table), to_cache(vp, table)
    for pos in (0, 1, 63, 64, 191, 192, 200, 3 * W + 70):
        k = rng.standard_normal((n_kv, hd)).astype(np.float32)
        v = rng.standard_normal((n_kv, hd)).astype(np.float32)
        before_k = kp.copy()
        append(kp, vp, table, k, v, pos)
        ref.kv_append(kc, vc, k, v, pos)
        assert np.array_equal(to_cache(kp, table), kc) and np.array_equal(to_cache(vp, table), vc)
        changed = np.argwhere(kp != before_k)
        slot = pos % W
        assert all(int(p) == table[slot // ref.PAGE_SLOTS] and int(r) == slot % ref.PAGE_SLOTS
                   for p, _, r, _ in changed)
    assert np.array_equal(kp[[1, 2, 4, 6]], pool[[1, 2, 4, 6]])   # pages nobody owns stay untouched


def test_paged_cache_bruteforce():
    pin_paged(ref.paged_to_cache, ref.paged_append)


def test_paged_attention_equals_contiguous():
    """A batch of sequences on one pool: each sequence's attention is the
    single-sequence attention of its gathered cache; identity tables reduce to
    a plain reshape of the pool."""
    import synth

    shape = synth.DecoderShape(n_layers=1, n_q_heads=4, n_kv_heads=2, head_dim=16, window=128)
    kp, vp = synth.page_pool(shape, 0, 5, 3)
    ident = np.array([0, 1], np.int32)
    assert np.array_equal(ref.paged_to_cache(kp, ident), kp[:2].transpose(1, 0, 2, 3).reshape(2, 128, 16))
    table = synth.page_table(2, 128, 5, 3)
    q = np.random.default_rng(4).standard_normal((2, 4, 16)).astype(np.float32)
    for s, pos in enumerate((40, 300)):
        kc, vc = ref.paged_to_cache(kp, table[s]), ref.paged_to_cache(vp, table[s])
        o = ref.gqa_attn(q[s], kc, vc, pos)
        assert np.allclose(o, ref.c_gqa_attn(q[s], kc, vc, pos), rtol=0, atol=1e-12)


def test_planted_mistakes_in_paging_are_caught():
    def row_major_pages(pool, table_row):             # page and row swapped
        n_pages, n_kv, ps, hd = pool.shape
        out = np.empty((n_kv, len(table_row) * ps, hd), pool.dtype)
        for slot in range(len(table_row) * ps):
            out[:, slot] = pool[table_row[slot % len(table_row)], :, slot // len(table_row)]
        return out

    def ignores_table(pool, table_row):
        return ref.paged_to_cache(pool, np.arange(len(table_row)))

    def append_wrong_row(k_pool, v_pool, table_row, k_new, v_new, pos):
        ref.paged_append(k_pool, v_pool, table_row, k_new, v_new, pos + 1)

    for bad in (row_major_pages, ignores_table):
        with pytest.raises(AssertionError):
            pin_paged(bad, ref.paged_append)
    with pytest.raises(AssertionError):
        pin_paged(ref.paged_to_cache, append_wrong_row)


# ------------------------------------------------------------------- RoPE
def pin_rope(rope):
    """Closed forms of the rotary embedding (reading R17)."""
    rng = np.random.default_rng(21)
    # a single pair (head_dim 2) turns by exactly pos radians (i = 0: frequency 1)
    for pos in (0, 1, 2, 7, 100):
        y = rope(np.array([1.0, 0.0]), pos, 10000.0, 2)
        assert np.allclose(y, [math.cos(pos), math.sin(pos)], rtol=0, atol=1e-12)
        y = rope(np.array([0.0, 1.0]), pos, 10000.0, 2)
        assert np.allclose(y, [-math.sin(pos), math.cos(pos)], rtol=0, atol=1e-12)
    # the frequency of pair i is theta^(-2i/hd): with hd 4, pair 1 turns by pos / theta^(1/2)
    y = rope(np.array([0.0, 0.0, 1.0, 0.0]), 3, 100.0, 4)
    assert np.allclose(y, [0.0, 0.0, math.cos(0.3), math.sin(0.3)], rtol=0, atol=1e-12)
    x = rng.standard_normal(3 * 8)
    assert np.array_equal(rope(x, 0, 1e6, 8), x)                          # position 0: identity
    assert np.array_equal(rope(x, 55, 0.0, 8), x)                         # off
    y = rope(x, 123, 1e4, 8)
    assert np.allclose(np.hypot(y[0::2], y[1::2]), np.hypot(x[0::2], x[1::2]), rtol=1e-12)   # pairs keep length
    # relative position: <R(m) q, R(n) k> depends on m - n only
    q, k = rng.standard_normal(16), rng.standard_normal(16)
    for m, n in ((5, 2), (40, 37), (1003, 1000)):
        assert abs(rope(q, m, 1e4, 16) @ rope(k, n, 1e4, 16) - rope(q, m - n, 1e4, 16) @ k) < 1e-9


def test_rope_closed_forms():
    pin_rope(ref.rope)


def test_decoder_layer_rope_off_is_unchanged_and_rope_at_pos0_is_identity():
    """rope_theta = 0 is the default layer; at position 0 RoPE changes nothing."""
    rng = np.random.default_rng(22)
    D, nq, nkv, hd, F, W = 8, 2, 1, 4, 6, 5
    Wd = {k: rng.standard_normal(s) for k, s in (("wq", (nq * hd, D)), ("wk", (nkv * hd, D)),
                                                  ("wv", (nkv * hd, D)), ("wo", (D, nq * hd)),
                                                  ("w1", (F, D)), ("w3", (F, D)), ("w2", (D, F)))}
    x = rng.standard_normal(D)
    kc = np.zeros((nkv, W, hd), np.uint16)
    for pos in (0, 3):
        a = ref.decoder_layer(x, Wd, kc.copy(), kc.copy(), pos, nq, nkv)
        b = ref.decoder_layer(x, Wd, kc.copy(), kc.copy(), pos, nq, nkv, rope_theta=0.0)
        assert np.array_equal(a["out"], b["out"])
        c = ref.decoder_layer(x, Wd, kc.copy(), kc.copy(), pos, nq, nkv, rope_theta=1e4)
        if pos == 0:
            assert np.array_equal(a["out"], c["out"])
        else:
            assert np.allclose(c["q"], ref.rope(Wd["wq"] @ a["n"], pos, 1e4, hd), rtol=0, atol=1e-12)
            assert not np.allclose(a["q"], c["q"])


def test_planted_mistakes_in_rope_are_caught():
    def half_split(x, pos, theta, hd):               # rotates (x[i], x[i + hd/2]) instead of adjacent pairs
        x = np.asarray(x, np.float64)
        y = x.reshape(-1, hd).copy()
        i = np.arange(hd // 2)
        ang = pos * np.power(float(theta), -2.0 * i / hd)
        a, b = y[:, :hd // 2].copy(), y[:, hd // 2:].copy()
        y[:, :hd // 2] = a * np.cos(ang) - b * np.sin(ang)
        y[:, hd // 2:] = a * np.sin(ang) + b * np.cos(ang)
        return y.reshape(x.shape)

    def wrong_sign(x, pos, theta, hd):
        return ref.rope(x, -pos, theta, hd)

    def wrong_frequency(x, pos, theta, hd):          # theta^(-i/hd)
        return ref.rope(x, pos, math.sqrt(theta), hd) if theta > 0 else np.asarray(x, np.float64).copy()

    for bad in (half_split, wrong_sign, wrong_frequency):
        with pytest.raises(AssertionError):
            pin_rope(bad)


# ------------------------------------------------------- streaming history
def pin_roll(roll):
    """After any sequence of chunks the history is exactly the last `window`
    positions seen, oldest first (a list model), for chunks shorter than,
    equal to and longer than the window."""
    for W, sizes in ((5, [2, 3, 1, 4]), (4, [4, 4]), (3, [7, 1, 2]), (750, [256, 256, 256, 256])):
        hist = -np.arange(W, 0, -1).reshape(W, 1)                 # positions -W .. -1
        seen = list(range(-W, 0))
        nxt = 0
        for n in sizes:
            new = np.arange(nxt, nxt + n).reshape(n, 1)
            nxt += n
            seen += list(range(nxt - n, nxt))
            hist = roll(hist, new, W)
            assert hist.shape == (W, 1) and hist[:, 0].tolist() == seen[-W:]


def test_roll_history_list_model():
    pin_roll(ref.roll_history)


def test_planted_mistakes_in_roll_are_caught():
    def first_rows(hist, new, window):
        both = np.concatenate([hist, new])
        return both[:window].copy()

    def new_first(hist, new, window):
        both = np.concatenate([new, hist])
        return both[both.shape[0] - window:].copy()

    for bad in (first_rows, new_first):
        with pytest.raises(AssertionError):
            pin_roll(bad)
