"""Parity of every libvox kernel with the CPU oracle on seeded inputs.

Bit-exact for dequantised weights, rolling-cache slots and bf16 cache bits;
otherwise max normalised error <= 2e-3 (error metric of the oracle module:
|y - y_ref| / (|x_m| |w_n|) for products, |o - o_ref| / (|p_h| |V_c|) for
attention).  Sizes span several tiles and a ragged tail; edge cases include
empty-like windows (one valid key), wrap-around and NaN/inf scales.
"""
import math

import numpy as np
import pytest

import synth
from oracle import ref

pytestmark = pytest.mark.gpu
TOL = 2e-3


@pytest.fixture(scope="module")
def env():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from bit_quantized_transformer_b200 import build

    build.build()
    from bit_quantized_transformer_b200 import vox as V
    from bit_quantized_transformer_b200 import workloads as WL

    return torch, V, WL


def np_of(t):
    return t.detach().cpu().numpy()


def bf16_bits(t):
    import torch

    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def check_status(V):
    torch = __import__("torch")
    torch.cuda.synchronize()
    assert V.vox_device_status(True) == 0


# ------------------------------------------------------------ pack/dequant
@pytest.mark.parametrize("n,k", [(16, 64), (37, 96), (130, 1280), (4096, 3072), (33, 32)])
def test_dequant_bitexact(env, n, k):
    torch, V, WL = env
    qs, d = synth.q4_blocks(n, k, 0, 7000 + n)
    packed, w = WL.pack_q4(qs, d, "cuda")
    out32 = torch.empty(n, k + 5, dtype=torch.float32, device="cuda")
    V.vox_q4_dequant(w, 0, n, out32, V.VOX_F32, k + 5)
    outbf = torch.empty(n, k, dtype=torch.bfloat16, device="cuda")
    V.vox_q4_dequant(w, 0, n, outbf, V.VOX_BF16, k)
    check_status(V)
    want32 = ref.c_dequant_f32(qs, d)
    got32 = np_of(out32)[:, :k]
    assert np.array_equal(got32.view(np.uint32), want32.view(np.uint32))
    assert np.array_equal(bf16_bits(outbf), ref.c_dequant_bf16(qs, d))
    # a row range in the middle
    r0, nr = n // 3, max(1, n // 4)
    part = torch.empty(nr, k, dtype=torch.float32, device="cuda")
    V.vox_q4_dequant(w, r0, nr, part, V.VOX_F32, k)
    assert np.array_equal(np_of(part).view(np.uint32), want32[r0:r0 + nr].view(np.uint32))


def test_dequant_handbuilt_and_special_scales(env):
    """The hand-worked blocks of tests/golden go through pack + dequant on the GPU."""
    torch, V, WL = env
    from test_oracle_pins import HANDBUILT, same_bits_or_nan

    qs = np.stack([c["qs"] for c in HANDBUILT])[:, None, :]
    d = np.array([[c["d"]] for c in HANDBUILT], np.uint16)
    n = len(HANDBUILT)
    _, w = WL.pack_q4(qs, d, "cuda")
    out = torch.empty(n, 32, dtype=torch.float32, device="cuda")
    V.vox_q4_dequant(w, 0, n, out, V.VOX_F32, 32)
    outbf = torch.empty(n, 32, dtype=torch.bfloat16, device="cuda")
    V.vox_q4_dequant(w, 0, n, outbf, V.VOX_BF16, 32)
    got = np_of(out)
    for i, c in enumerate(HANDBUILT):
        assert same_bits_or_nan(got[i], c["w"]), c["name"]
    assert np.array_equal(bf16_bits(outbf), ref.c_dequant_bf16(qs, d))


def test_dequant_bf16_ties(env):
    torch, V, WL = env
    rows = [(0x3C04, 0x3F80), (0x3C0C, 0x3F82), (0x3C05, 0x3F81), (0xBC04, 0xBF80)]
    qs = np.full((len(rows), 1, 16), 0x99, np.uint8)
    d = np.array([[a] for a, _ in rows], np.uint16)
    _, w = WL.pack_q4(qs, d, "cuda")
    out = torch.empty(len(rows), 32, dtype=torch.bfloat16, device="cuda")
    V.vox_q4_dequant(w, 0, len(rows), out, V.VOX_BF16, 32)
    assert np.array_equal(bf16_bits(out), np.array([[b] * 32 for _, b in rows], np.uint16))


def test_gate_up_pack_order(env):
    torch, V, WL = env
    F, k = 24, 64
    q1, d1 = synth.q4_blocks(F, k, 0, 8101)
    q3, d3 = synth.q4_blocks(F, k, 0, 8103)
    _, w = WL.pack_q4(np.concatenate([q1, q3]), np.concatenate([d1, d3]), "cuda", V.VOX_PACK_GATE_UP)
    out = torch.empty(2 * F, k, dtype=torch.float32, device="cuda")
    V.vox_q4_dequant(w, 0, 2 * F, out, V.VOX_F32, k)
    got = np_of(out)
    W1, W3 = ref.c_dequant_f32(q1, d1), ref.c_dequant_f32(q3, d3)
    for j in range(F // 8):
        assert np.array_equal(got[16 * j:16 * j + 8], W1[8 * j:8 * j + 8])
        assert np.array_equal(got[16 * j + 8:16 * j + 16], W3[8 * j:8 * j + 8])


# -------------------------------------------------------------------- GEMV
def run_gemv(env, qs, d, x, ep=None, flags=0, ldy=None, y_init=None):
    torch, V, WL = env
    n = qs.shape[0]
    k = qs.shape[1] * 32
    m = x.shape[0]
    packed, w = WL.pack_q4(qs, d, "cuda", flags)
    xt = WL.to_dev(x, "cuda")
    ldy = n if ldy is None else ldy
    y = WL.to_dev(y_init, "cuda") if y_init is not None else torch.full((m, ldy), float("nan"), device="cuda")
    wsb = V.vox_q4_gemv_workspace(w, m, ep)
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    V.vox_q4_gemv(w, xt, m, k, y, ldy, ep, ws, wsb)
    check_status(V)
    return np_of(y), ws


@pytest.mark.parametrize("n,k,m", [(4096, 3072, 1), (37, 96, 1), (100, 1280, 3), (6144, 3072, 1),
                                   (3072, 9216, 8), (3072, 4096, 2), (18432, 3072, 1), (16, 32, 5),
                                   (1024, 3072, 4)])
def test_gemv_parity(env, n, k, m):
    qs, d = synth.q4_blocks(n, k, 0, 9000 + n + k)
    x = synth.activations(m, k, 0, 9500 + m)
    y, _ = run_gemv(env, qs, d, x)
    y_ref = ref.c_matvec(qs, d, x)
    err = ref.gemv_error(y, y_ref, x, ref.q4_weights(qs, d))
    assert err <= TOL, err


def test_gemv_special_inputs(env):
    n, k = 48, 256
    qs, d = synth.q4_blocks(n, k, 0, 9901)
    y, _ = run_gemv(env, qs, d, np.zeros((2, k), np.float32))
    assert np.all(y == 0.0)
    x = np.zeros((1, k), np.float32)
    x[0, 77] = 1.0
    y, _ = run_gemv(env, qs, d, x)
    W = ref.q4_weights(qs, d)
    assert ref.gemv_error(y, W[:, 77][None], x, W) <= TOL
    # large-magnitude activations (outside fp16 range before the exact power-of-two scaling)
    xl = synth.activations(1, k, 0, 9902) * 3.0e6
    y, _ = run_gemv(env, qs, d, xl)
    assert ref.gemv_error(y, ref.c_matvec(qs, d, xl), xl, W) <= TOL
    xs = synth.activations(1, k, 0, 9903) * 1.0e-6
    y, _ = run_gemv(env, qs, d, xs)
    assert ref.gemv_error(y, ref.c_matvec(qs, d, xs), xs, W) <= TOL


def test_gemv_rmsnorm_residual_gelu(env):
    torch, V, WL = env
    n, k, m = 3072, 3072, 2
    qs, d = synth.q4_blocks(n, k, 0, 9911)
    x = synth.activations(m, k, 0, 9912) * 3.0
    W = ref.q4_weights(qs, d)
    xn = ref.rmsnorm(x)
    ep = V.vox_epilogue(op=V.VOX_EP_NONE, rmsnorm=1, eps=1e-5)
    y, _ = run_gemv(env, qs, d, x, ep)
    assert ref.gemv_error(y, xn @ W.T, xn, W) <= TOL
    res = synth.activations(m, n, 0, 9913)
    rt = WL.to_dev(res, "cuda")
    ep = V.vox_epilogue(op=V.VOX_EP_RESIDUAL, residual=rt.data_ptr(), ldr=n)
    y, _ = run_gemv(env, qs, d, x, ep)
    assert ref.gemv_error(y - res, x.astype(np.float64) @ W.T, x, W) <= TOL
    ep = V.vox_epilogue(op=V.VOX_EP_GELU)
    y, _ = run_gemv(env, qs, d, x, ep)
    want = ref.gelu(x.astype(np.float64) @ W.T)
    # gelu is 1.13-Lipschitz: the product's bound carries over
    assert ref.gemv_error(y, want, x, W) <= TOL


def test_gemv_silu_mul(env):
    torch, V, WL = env
    F, k, m = 9216, 3072, 1
    q1, d1 = synth.q4_blocks(F, k, 0, 9921)
    q3, d3 = synth.q4_blocks(F, k, 0, 9923)
    x = synth.activations(m, k, 0, 9924)
    ep = V.vox_epilogue(op=V.VOX_EP_SILU_MUL, rmsnorm=1, eps=1e-5)
    y, _ = run_gemv(env, np.concatenate([q1, q3]), np.concatenate([d1, d3]), x, ep, V.VOX_PACK_GATE_UP, ldy=F)
    xn = ref.rmsnorm(x)
    g = xn @ ref.q4_weights(q1, d1).T
    u = xn @ ref.q4_weights(q3, d3).T
    want = ref.silu(g) * u
    # first-order error: |silu'(g)| |u| e_g + |silu(g)| e_u, each e <= TOL |x| |w_row|
    w1n = np.linalg.norm(ref.q4_weights(q1, d1), axis=1)
    w3n = np.linalg.norm(ref.q4_weights(q3, d3), axis=1)
    xnn = np.linalg.norm(xn)
    bound = 1.1 * np.abs(u) * xnn * w1n + np.abs(ref.silu(g)) * xnn * w3n
    assert np.all(np.abs(y[0] - want[0]) <= TOL * bound[0] + 1e-30)


def test_gemv_kv_append_epilogue(env):
    torch, V, WL = env
    QD, n_kv, hd, W = 256, 2, 64, 7
    n, k = QD + 2 * n_kv * hd, 512
    qs, d = synth.q4_blocks(n, k, 0, 9931)
    x = synth.activations(2, k, 0, 9932)           # two tokens at positions 12, 13
    kc = torch.zeros(n_kv, W, hd, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    ep = V.vox_epilogue(op=V.VOX_EP_KV_APPEND, k_cache=kc.data_ptr(), v_cache=vc.data_ptr(), n_kv_heads=n_kv,
                        head_dim=hd, window=W, q_rows=QD, pos=12)
    y, _ = run_gemv(env, qs, d, x, ep)
    Wd = ref.q4_weights(qs, d)
    assert ref.gemv_error(y, x.astype(np.float64) @ Wd.T, x, Wd) <= TOL
    kb, vb = bf16_bits(kc), bf16_bits(vc)
    for i, p in enumerate((12, 13)):
        s = p % W
        kk = ref.f32_to_bf16(y[i, QD:QD + n_kv * hd]).reshape(n_kv, hd)
        vv = ref.f32_to_bf16(y[i, QD + n_kv * hd:]).reshape(n_kv, hd)
        assert np.array_equal(kb[:, s], kk) and np.array_equal(vb[:, s], vv)
    untouched = [s for s in range(W) if s not in (12 % W, 13 % W)]
    assert np.all(kb[:, untouched] == 0) and np.all(vb[:, untouched] == 0)


def test_gemv_argmax(env):
    torch, V, WL = env
    n, k, m = 131072, 3072, 2
    qs, d = synth.q4_blocks(n, k, 0, 9941)
    x = synth.activations(m, k, 0, 9942)
    am = torch.full((m,), -1, dtype=torch.int32, device="cuda")
    ep = V.vox_epilogue(op=V.VOX_EP_ARGMAX, rmsnorm=1, eps=1e-5, argmax=am.data_ptr())
    y, ws = run_gemv(env, qs, d, x, ep)
    got = np_of(am)
    for i in range(m):
        assert got[i] == int(np.argmax(y[i]))               # same precision: the kernel's logits
    # logits on sampled rows (including the winners) against the oracle
    xn = ref.rmsnorm(x)
    rows = np.unique(np.concatenate([got, np.random.default_rng(0).integers(0, n, 256)]))
    assert ref.gemv_error(y[:, rows], xn @ ref.q4_weights(qs[rows], d[rows]).T, xn,
                          ref.q4_weights(qs[rows], d[rows])) <= TOL
    # with a clear margin the winner is the oracle's winner
    yr = ref.c_matvec(qs, d, xn.astype(np.float32))
    for i in range(m):
        top = np.sort(yr[i])[-2:]
        if top[1] - top[0] > 1e-3 * abs(top[1]):
            assert got[i] == int(np.argmax(yr[i]))


def test_gemv_shared_workspace_across_shapes(env):
    """Consecutive calls on different matrices share one workspace (as the
    decoder step does): the arrival counters each call leaves behind must not
    disturb the next one."""
    torch, V, WL = env
    k = 3072
    shapes = [(6144, 9951), (18432, 9952), (1024, 9953), (6144, 9951)]
    ws = None
    for n, tid in shapes:
        qs, d = synth.q4_blocks(n, k, 0, tid)
        x = synth.activations(1, k, 0, tid + 1)
        packed, w = WL.pack_q4(qs, d, "cuda")
        if ws is None:
            wsb = max(V.vox_q4_gemv_workspace(V.weight(packed, nn, k), 1, None) for nn, _ in shapes)
            ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
        y = torch.full((1, n), float("nan"), device="cuda")
        V.vox_q4_gemv(w, WL.to_dev(x, "cuda"), 1, k, y, n, None, ws, ws.numel())
        check_status(V)
        err = ref.gemv_error(np_of(y), ref.c_matvec(qs, d, x), x, ref.q4_weights(qs, d))
        assert err <= TOL, (n, err)


def test_gemv_argmax_ties_lowest_index(env):
    torch, V, WL = env
    n, k = 4096, 64
    qs = np.full((n, 2, 16), 0x88, np.uint8)                # all weights 0 -> all logits 0
    d = np.full((n, 2), 0x3C00, np.uint16)
    qs[777] = 0x99; qs[3000] = 0x99                          # rows 777 and 3000 tie at the max
    x = np.ones((1, k), np.float32)
    am = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    ep = V.vox_epilogue(op=V.VOX_EP_ARGMAX, argmax=am.data_ptr())
    run_gemv(env, qs, d, x, ep)
    assert int(am.item()) == 777
    run_gemv(env, qs, d, x, ep)                              # second call on a fresh workspace
    assert int(am.item()) == 777


# --------------------------------------------------------- rolling append
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_kv_append_bitexact(env, dtype):
    torch, V, WL = env
    n_kv, hd, W = 8, 128, 5
    kc = torch.zeros(n_kv, W, hd, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    kc_ref = np.zeros((n_kv, W, hd), np.uint16)
    vc_ref = kc_ref.copy()
    rng = np.random.default_rng(3)
    for p in range(3 * W + 2):
        kn = rng.standard_normal((n_kv, hd)).astype(np.float32)
        vn = rng.standard_normal((n_kv, hd)).astype(np.float32)
        if dtype == "f32":
            V.vox_kv_append_rolling(kc, vc, WL.to_dev(kn, "cuda"), WL.to_dev(vn, "cuda"), V.VOX_F32, n_kv, hd, W, p)
            ref.c_kv_append(kc_ref, vc_ref, kn, vn, p)
        else:
            kbits, vbits = ref.f32_to_bf16(kn), ref.f32_to_bf16(vn)
            V.vox_kv_append_rolling(kc, vc, WL.bf16_dev(kbits, "cuda"), WL.bf16_dev(vbits, "cuda"), V.VOX_BF16,
                                    n_kv, hd, W, p)
            kc_ref[:, p % W] = kbits
            vc_ref[:, p % W] = vbits
        assert np.array_equal(bf16_bits(kc), kc_ref) and np.array_equal(bf16_bits(vc), vc_ref)


# ------------------------------------------------------- matmul dispatch
@pytest.mark.parametrize("m", [1, 8, 9, 16, 64])
@pytest.mark.parametrize("epi", ["none", "rms_gelu", "residual"])
def test_matmul_dispatch(env, m, epi):
    """vox_q4_matmul at either side of the GEMV / GEMM crossover, fp32 in and
    out, with the epilogues both kernels share; checked against the oracle on
    the fp32 input (the GEMM side's bf16 rounding of x is the kernel's error)."""
    torch, V, WL = env
    n, k = 384, 1280
    qs, d = synth.q4_blocks(n, k, 0, 9500 + m)
    x = synth.activations(m, k, 0, 9600 + m) * 3.0
    res = synth.activations(m, n, 0, 9700 + m)
    packed, w = WL.pack_q4(qs, d, "cuda")
    W = ref.q4_weights(qs, d)
    ep = None
    xr = x.astype(np.float64)
    if epi == "rms_gelu":
        ep = V.vox_epilogue(op=V.VOX_EP_GELU, rmsnorm=1, eps=1e-5)
        xr = ref.rmsnorm(xr)
    elif epi == "residual":
        rt = WL.to_dev(res, "cuda")
        ep = V.vox_epilogue(op=V.VOX_EP_RESIDUAL, residual=rt.data_ptr(), ldr=n)
    y = torch.full((m, n), float("nan"), device="cuda")
    wsb = V.vox_q4_matmul_workspace(w, m, ep)
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    V.vox_q4_matmul(w, WL.to_dev(x, "cuda"), m, k, y, n, ep, ws, wsb)
    check_status(V)
    got = np_of(y).astype(np.float64)
    want = xr @ W.T
    if epi == "rms_gelu":
        got_lin, want = got, ref.gelu(want)
        err = ref.gemv_error(got_lin, want, xr, W)
    elif epi == "residual":
        err = ref.gemv_error(got - res, want, xr, W)
    else:
        err = ref.gemv_error(got, want, xr, W)
    assert err <= TOL, err


# -------------------------------------------------------------- attention
def attn_case(env, n_q, n_kv, hd, W, pos, seed=0, nan_fill=False):
    torch, V, WL = env
    kb = synth.bf16_normal((n_kv, W, hd), seed, 11)
    vb = synth.bf16_normal((n_kv, W, hd), seed, 12)
    if nan_fill:                                    # slots never written hold NaN bits
        nv = min(pos + 1, W)
        kb = kb.copy(); vb = vb.copy()
        kb[:, nv:] = 0x7FC1; vb[:, nv:] = 0x7FC1
    q = synth.activations(n_q, hd, seed, 13) * 2.0
    kc, vc = WL.bf16_dev(kb, "cuda"), WL.bf16_dev(vb, "cuda")
    out = torch.full((n_q, hd), float("nan"), device="cuda")
    wsb = V.vox_gqa_decode_attn_workspace(n_q, n_kv, hd, W)
    ws = torch.full((wsb,), 0xFF, dtype=torch.uint8, device="cuda")    # no initial contents needed
    V.vox_gqa_decode_attn(WL.to_dev(q, "cuda"), kc, vc, out, n_q, n_kv, hd, W, pos, 1.0 / math.sqrt(hd), ws, wsb)
    check_status(V)
    o = np_of(out)
    o_ref = ref.c_gqa_attn(q, kb, vb, pos)
    P = ref.attn_probs(q, kb, pos)
    nv = min(pos + 1, W)
    err = ref.attn_error(o, o_ref, P, ref.bf16_to_f64(vb[:, :nv]), n_q // n_kv)
    return err, o, o_ref


@pytest.mark.parametrize("pos", [0, 1, 63, 64, 200, 1024, 8191, 8492, 3 * 8192 + 5])
def test_attention_decoder_shape(env, pos):
    err, o, _ = attn_case(env, 32, 8, 128, 8192, pos)
    assert np.all(np.isfinite(o))
    assert err <= TOL, err


@pytest.mark.parametrize("n_q,n_kv,W,pos", [(8, 8, 100, 250), (16, 2, 257, 40), (4, 1, 65, 64), (64, 8, 300, 299),
                                            (8, 1, 1, 7)])
def test_attention_groups_and_windows(env, n_q, n_kv, W, pos):
    err, o, _ = attn_case(env, n_q, n_kv, 128, W, pos)
    assert np.all(np.isfinite(o))
    assert err <= TOL, err


def test_attention_single_key_is_exact_v(env):
    err, o, o_ref = attn_case(env, 32, 8, 128, 8192, 0)
    assert np.array_equal(o, o_ref.astype(np.float32))


def test_attention_ignores_unwritten_slots(env):
    err, o, _ = attn_case(env, 32, 8, 128, 8192, 300, nan_fill=True)
    assert np.all(np.isfinite(o)) and err <= TOL


# ------------------------------------------------------- window attention
def test_window_attention_encoder_shape(env):
    torch, V, WL = env
    nh, hd, W, nhist, nq = 32, 40, 750, 750, 256
    D = nh * hd
    khb = synth.bf16_normal((nhist, D), 0, 21)
    vhb = synth.bf16_normal((nhist, D), 0, 22)
    qkvb = synth.bf16_normal((nq, 3 * D), 0, 23)
    out = torch.full((nq, D), float("nan"), device="cuda")
    qkv = WL.bf16_dev(qkvb, "cuda")
    V.vox_window_attn(qkv, 3 * D, WL.bf16_dev(khb, "cuda"), WL.bf16_dev(vhb, "cuda"), D, nhist,
                      qkv[:, D:], qkv[:, 2 * D:], 3 * D, nq, out, V.VOX_F32, D, nh, hd, W, 1.0 / math.sqrt(hd))
    check_status(V)
    o = np_of(out)
    Q = ref.bf16_to_f64(qkvb[:, :D])
    K = np.concatenate([ref.bf16_to_f64(khb), ref.bf16_to_f64(qkvb[:, D:2 * D])])
    Vv = np.concatenate([ref.bf16_to_f64(vhb), ref.bf16_to_f64(qkvb[:, 2 * D:])])
    rows = list(range(0, nq, 17)) + [nq - 1]
    o_ref = np.concatenate([ref.window_attn(Q[i:i + 1], K, Vv, nhist + i, W, nh, hd) for i in rows])
    err = 0.0
    for ii, i in enumerate(rows):
        p = nhist + i
        lo = max(0, p - W + 1)
        for h in range(nh):
            sl = slice(h * hd, (h + 1) * hd)
            s = (K[lo:p + 1, sl] @ Q[i, sl]) / math.sqrt(hd)
            pr = np.exp(s - s.max()); pr /= pr.sum()
            den = np.linalg.norm(pr) * np.linalg.norm(Vv[lo:p + 1, sl], axis=0)
            err = max(err, float(np.max(np.abs(o[i, sl] - o_ref[ii, sl]) / den)))
    assert err <= TOL, err


def test_window_attention_short_history(env):
    torch, V, WL = env
    nh, hd, W, nhist, nq = 2, 40, 5, 3, 70
    D = nh * hd
    khb = synth.bf16_normal((nhist, D), 1, 31)
    vhb = synth.bf16_normal((nhist, D), 1, 32)
    qkvb = synth.bf16_normal((nq, 3 * D), 1, 33)
    out = torch.full((nq, D), float("nan"), device="cuda")
    qkv = WL.bf16_dev(qkvb, "cuda")
    V.vox_window_attn(qkv, 3 * D, WL.bf16_dev(khb, "cuda"), WL.bf16_dev(vhb, "cuda"), D, nhist,
                      qkv[:, D:], qkv[:, 2 * D:], 3 * D, nq, out, V.VOX_F32, D, nh, hd, W, 1.0 / math.sqrt(hd))
    check_status(V)
    Q = ref.bf16_to_f64(qkvb[:, :D])
    K = np.concatenate([ref.bf16_to_f64(khb), ref.bf16_to_f64(qkvb[:, D:2 * D])])
    Vv = np.concatenate([ref.bf16_to_f64(vhb), ref.bf16_to_f64(qkvb[:, 2 * D:])])
    o_ref = ref.window_attn(Q, K, Vv, nhist, W, nh, hd)
    assert np.max(np.abs(np_of(out) - o_ref)) <= TOL * np.max(np.abs(Vv))


# ------------------------------------------------------------------- GEMM
@pytest.mark.parametrize("n,k,m", [(256, 128, 16), (1280, 1280, 256), (3840, 1280, 256), (1280, 5120, 256),
                                   (3072, 5120, 64), (130, 320, 37), (6144, 3072, 16), (5120, 1280, 100),
                                   (48, 192, 20)])
def test_gemm_parity(env, n, k, m):
    torch, V, WL = env
    qs, d = synth.q4_blocks(n, k, 0, 12000 + n + k)
    xb = synth.bf16_normal((m, k), 0, 12500 + m)
    packed, w = WL.pack_q4(qs, d, "cuda")
    y = torch.full((m, n), float("nan"), device="cuda")
    V.vox_q4_gemm(w, WL.bf16_dev(xb, "cuda"), V.VOX_BF16, m, k, y, V.VOX_F32, n)
    check_status(V)
    x = ref.bf16_to_f64(xb)
    Wd = ref.q4_weights(qs, d)
    err = ref.gemv_error(np_of(y), x @ Wd.T, x, Wd)
    assert err <= TOL, err


def test_gemm_weights_round_once(env):
    """With one-hot activation rows (X = I), the GEMM's output is the bf16
    weight tile the kernel staged in shared memory, widened exactly: it must
    equal vox_q4_dequant's bf16 weights (round-to-nearest-even of the exact
    (q - 8) d) bit for bit, including scales whose products need rounding."""
    torch, V, WL = env
    n, k = 256, 128
    qs, d = synth.q4_blocks(n, k, 0, 9901)
    d = d.copy()
    d[::3] = synth.fp16_bits(np.linspace(0.0011, 0.0117, d[::3].size)).reshape(d[::3].shape)   # 11-bit scales
    packed, w = WL.pack_q4(qs, d, "cuda")
    X = torch.eye(k, dtype=torch.bfloat16, device="cuda")
    Y = torch.full((k, n), float("nan"), dtype=torch.float32, device="cuda")
    V.vox_q4_gemm(w, X, V.VOX_BF16, k, k, Y, V.VOX_F32, n)
    Wb = torch.empty(n, k, dtype=torch.bfloat16, device="cuda")
    V.vox_q4_dequant(w, 0, n, Wb, V.VOX_BF16, k)
    check_status(V)
    got = Y.cpu().numpy().T                                  # [n][k]
    want = ref.bf16_to_f64(bf16_bits(Wb)).astype(np.float32)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
    assert np.array_equal(bf16_bits(Wb), ref.c_dequant_bf16(qs, d))


def test_gemm_epilogues(env):
    torch, V, WL = env
    n, k, m = 1280, 5120, 256
    qs, d = synth.q4_blocks(n, k, 0, 13001)
    xb = synth.bf16_normal((m, k), 0, 13002)
    res = synth.activations(m, n, 0, 13003)
    packed, w = WL.pack_q4(qs, d, "cuda")
    x = ref.bf16_to_f64(xb)
    Wd = ref.q4_weights(qs, d)
    yref = x @ Wd.T
    y = WL.to_dev(res, "cuda")
    ep = V.vox_epilogue(op=V.VOX_EP_RESIDUAL, residual=y.data_ptr(), ldr=n)
    V.vox_q4_gemm(w, WL.bf16_dev(xb, "cuda"), V.VOX_BF16, m, k, y, V.VOX_F32, n, ep)
    check_status(V)
    assert ref.gemv_error(np_of(y) - res, yref, x, Wd) <= TOL
    yb = torch.zeros((m, n), dtype=torch.bfloat16, device="cuda")
    ep = V.vox_epilogue(op=V.VOX_EP_GELU)
    V.vox_q4_gemm(w, WL.bf16_dev(xb, "cuda"), V.VOX_BF16, m, k, yb, V.VOX_BF16, n, ep)
    check_status(V)
    got = ref.bf16_to_f64(bf16_bits(yb))
    assert ref.gemv_error(got, ref.gelu(yref), x, Wd) <= TOL


# ---------------------------------------------------------------- RMSNorm
def test_rmsnorm(env):
    torch, V, WL = env
    x = synth.activations(5, 1280, 0, 14001) * 4.0
    out = torch.empty(5, 1280, device="cuda")
    V.vox_rmsnorm(WL.to_dev(x, "cuda"), 5, 1280, 1280, 1e-5, None, out, V.VOX_F32, 1280)
    check_status(V)
    np.testing.assert_allclose(np_of(out), ref.rmsnorm(x), rtol=1e-5, atol=1e-6)


@pytest.mark.gpu
@pytest.mark.parametrize("n", [1280, 3072, 5120, 1283])
def test_rmsnorm_weight_bf16(env, n):
    """RMSNorm with a weight into bf16 rows: the 16-byte path (n a multiple of
    4, one or two float4 per thread) and the element path (n = 1283).  Each
    value is within one bf16 rounding of the oracle's."""
    torch, V, WL = env
    m = 7
    x = synth.activations(m, n, 0, 14002) * 3.0
    g = synth.activations(1, n, 0, 14003)[0] + 1.5
    out = torch.empty(m, n, dtype=torch.bfloat16, device="cuda")
    V.vox_rmsnorm(WL.to_dev(x, "cuda"), m, n, n, 1e-5, WL.to_dev(g, "cuda"), out, V.VOX_BF16, n)
    check_status(V)
    want = ref.rmsnorm(x, g=g)
    got = out.float().cpu().numpy().astype(np.float64)
    np.testing.assert_allclose(got, want, rtol=2.0 ** -8, atol=1e-30)


# ------------------------------------------------------------------- RoPE
@pytest.mark.parametrize("pos,theta", [(0, 1e6), (7, 1e4), (8191, 1e6), (100000, 1e6), (123457, 500.0)])
def test_gemv_kv_append_rope(env, pos, theta):
    """The QKV epilogue with the rotary embedding: the GPU's q and k rows,
    turned back by the oracle's inverse rotation, match the plain product;
    the cache holds bf16 of the rotated k rows (two tokens, positions pos
    and pos + 1)."""
    torch, V, WL = env
    n_q, n_kv, hd, W, k, m = 4, 2, 128, 256, 384, 2
    QD, KVD = n_q * hd, n_kv * hd
    n = QD + 2 * KVD
    qs, d = synth.q4_blocks(n, k, 0, 8200)
    packed, w = WL.pack_q4(qs, d, "cuda")
    x = synth.activations(m, k, 0, 8201)
    kc = torch.zeros(n_kv, W, hd, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    y = torch.full((m, n), float("nan"), device="cuda")
    e = V.vox_epilogue(op=V.VOX_EP_KV_APPEND, k_cache=kc.data_ptr(), v_cache=vc.data_ptr(), n_kv_heads=n_kv,
                       head_dim=hd, window=W, q_rows=QD, pos=pos, rope_theta=theta)
    wsb = V.vox_q4_gemv_workspace(w, m, e)
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    V.vox_q4_gemv(w, WL.to_dev(x, "cuda"), m, k, y, n, e, ws, wsb)
    check_status(V)
    yv = np_of(y).astype(np.float64)
    Wm = ref.q4_weights(qs, d)
    y_ref = x.astype(np.float64) @ Wm.T
    back = yv.copy()
    for i in range(m):
        back[i, :QD] = ref.rope(yv[i, :QD], -(pos + i), theta, hd)
        back[i, QD:QD + KVD] = ref.rope(yv[i, QD:QD + KVD], -(pos + i), theta, hd)
    assert ref.gemv_error(back, y_ref, x, Wm) <= TOL
    if pos > 0:                                        # the rotation did happen
        assert ref.gemv_error(yv, y_ref, x, Wm) > 10 * TOL
    kb = bf16_bits(kc)
    for i in range(m):
        assert np.array_equal(kb[:, (pos + i) % W], ref.f32_to_bf16(np_of(y)[i, QD:QD + KVD]).reshape(n_kv, hd))


@pytest.mark.parametrize("splits,bn", [(1, 64), (2, 128), (3, 256), (7, 128), (8, 32)])
def test_gemm_split_k(env, monkeypatch, splits, bn):
    """The GEMM with K split over a cluster of CTAs (partial tiles summed in
    rank order through distributed shared memory): within tolerance of the
    oracle for the residual and GELU epilogues, ragged rows and tokens, and
    identical bits on a second call."""
    torch, V, WL = env
    monkeypatch.setenv("VOX_GEMM_SPLITS", str(splits))
    monkeypatch.setenv("VOX_GEMM_BN", str(bn))
    n, k, m = 1296, 1280, 200
    qs, d = synth.q4_blocks(n, k, 0, 13101)
    xb = synth.bf16_normal((m, k), 0, 13102)
    res = synth.activations(m, n, 0, 13103)
    packed, w = WL.pack_q4(qs, d, "cuda")
    x = ref.bf16_to_f64(xb)
    Wd = ref.q4_weights(qs, d)
    yref = x @ Wd.T
    xd = WL.bf16_dev(xb, "cuda")
    outs = []
    for _ in range(2):
        y = WL.to_dev(res, "cuda")
        ep = V.vox_epilogue(op=V.VOX_EP_RESIDUAL, residual=y.data_ptr(), ldr=n)
        V.vox_q4_gemm(w, xd, V.VOX_BF16, m, k, y, V.VOX_F32, n, ep)
        check_status(V)
        outs.append(np_of(y))
    assert np.array_equal(outs[0].view(np.uint32), outs[1].view(np.uint32))
    assert ref.gemv_error(outs[0] - res, yref, x, Wd) <= TOL
    yb = torch.zeros((m, n), dtype=torch.bfloat16, device="cuda")
    V.vox_q4_gemm(w, xd, V.VOX_BF16, m, k, yb, V.VOX_BF16, n, V.vox_epilogue(op=V.VOX_EP_GELU))
    check_status(V)
    assert ref.gemv_error(ref.bf16_to_f64(bf16_bits(yb)), ref.gelu(yref), x, Wd) <= TOL
