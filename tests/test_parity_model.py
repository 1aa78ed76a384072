"""Parity of the composed paths (vox_decoder_step, vox_encoder_chunk) with the
oracle, kernel by kernel on the GPU's own inputs to each kernel (teacher
forcing, so errors do not compound), at the benchmark's full sizes.

* one decoder layer, KV length 1024 (every kernel of the layer checked);
* the full 26-layer step with the cache filled to 8192 + 300 (wrapped): the
  last layer's attention, FFN and residual, the LM head on sampled rows and
  the argmax;
* each decoder check for both forms of the step: the single persistent
  launch and the per-kernel launch sequence, and small shapes on which nearly
  every tile of the persistent step is cut between warps and CTAs;
* one encoder layer + the adapter GEMM at M = 256, and the last layer of the
  full 32-layer chunk, each kernel on that layer's own inputs (a tap of the
  layer's input and mid-layer residual).
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


def bits(t):
    import torch

    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def gemv_err(y, x, qs, d, extra=None):
    W = ref.q4_weights(qs, d)
    want = np.atleast_2d(x).astype(np.float64) @ W.T
    if extra is not None:
        want = want + extra
    return ref.gemv_error(np.atleast_2d(y), want, x, W)


def check_layer_tail(shape, layer, dm, seed, pos_written):
    """Attention, FFN and the final residual of `layer` from the GPU buffers."""
    D, QD, KVD, F = shape.dim, shape.q_dim, shape.kv_dim, shape.ffn
    w = synth.decoder_layer_weights(shape, layer, seed)
    qkv = np_of(dm.qkv)
    kc, vc = bits(dm.k_cache[layer]), bits(dm.v_cache[layer])
    # the rolling append wrote bf16 of this step's k and v at slot pos mod W
    slot = pos_written % dm.W
    assert np.array_equal(kc[:, slot], ref.f32_to_bf16(qkv[QD:QD + KVD]).reshape(shape.n_kv_heads, -1))
    assert np.array_equal(vc[:, slot], ref.f32_to_bf16(qkv[QD + KVD:]).reshape(shape.n_kv_heads, -1))
    k0, v0 = synth.decoder_layer_cache(shape, layer, seed, dm.W)
    others = np.ones(dm.W, bool)
    others[slot] = False
    assert np.array_equal(kc[:, others], k0[:, others]) and np.array_equal(vc[:, others], v0[:, others])
    # attention on the GPU's q and caches
    q = qkv[:QD].reshape(shape.n_q_heads, shape.head_dim)
    o = np_of(dm.attn).reshape(shape.n_q_heads, shape.head_dim)
    o_ref = ref.c_gqa_attn(q, kc, vc, pos_written)
    nv = min(pos_written + 1, dm.W)
    err_attn = ref.attn_error(o, o_ref, ref.attn_probs(q, kc, pos_written), ref.bf16_to_f64(vc[:, :nv]),
                              shape.n_q_heads // shape.n_kv_heads)
    assert err_attn <= TOL, err_attn
    # FFN on the GPU's h: a = silu(W1 n2) * (W3 n2)
    h = np_of(dm.h)
    n2 = ref.rmsnorm(h)
    g = n2 @ ref.q4_weights(*w["w1"]).T
    u = n2 @ ref.q4_weights(*w["w3"]).T
    a = np_of(dm.act)
    w1n = np.linalg.norm(ref.q4_weights(*w["w1"]), axis=1)
    w3n = np.linalg.norm(ref.q4_weights(*w["w3"]), axis=1)
    bound = 1.1 * np.abs(u) * np.linalg.norm(n2) * w1n + np.abs(ref.silu(g)) * np.linalg.norm(n2) * w3n
    assert np.all(np.abs(a - ref.silu(g) * u) <= TOL * bound)
    # x_out = h + W2 a
    x_out = np_of(dm.x)
    err_w2 = gemv_err((x_out - h)[None], a[None], *w["w2"])
    assert err_w2 <= TOL, err_w2
    return w, o


FORMS = ["persistent", "kernels", "fused"]


def run_step(dm, form, stream=None):
    """One decoder step in the given form: one persistent launch
    (vox_decoder_step), the per-kernel launch sequence, or persistent
    projection segments between attention launches (vox_decoder_step_fused)."""
    if form == "persistent":
        dm.step(stream)
    elif form == "fused":
        dm.step_fused(stream)
    else:
        dm.step_kernels(stream)


@pytest.mark.parametrize("form", FORMS)
def test_decoder_layer_kv1024(env, form):
    torch, V, WL = env
    shape = synth.DecoderShape()
    tok = 4242
    dm = WL.DecoderModel(shape, seed=0, n_layers=1, filled=1024, token=tok)
    run_step(dm, form)
    torch.cuda.synchronize()
    assert V.vox_device_status(True) == 0
    assert int(dm.pos.item()) == 1025
    D, QD, KVD = shape.dim, shape.q_dim, shape.kv_dim
    # x0 = embedding row, exact
    eq, ed = synth.q4_blocks(shape.vocab, D, 0, synth.EMB_ID)
    x0 = ref.c_dequant_f32(eq, ed, row0=tok, nrows=1)[0]
    # QKV on the GPU's (exact) x0 with the RMSNorm prologue
    w = synth.decoder_layer_weights(shape, 0, 0)
    qs = np.concatenate([w["wq"][0], w["wk"][0], w["wv"][0]])
    ds = np.concatenate([w["wq"][1], w["wk"][1], w["wv"][1]])
    n0 = ref.rmsnorm(x0)
    err_qkv = gemv_err(np_of(dm.qkv)[None], n0[None], qs, ds)
    assert err_qkv <= TOL, err_qkv
    w, o = check_layer_tail(shape, 0, dm, 0, 1024)
    # Wo + residual on the GPU's attention output
    err_wo = gemv_err((np_of(dm.h) - x0)[None], np_of(dm.attn)[None], *w["wo"])
    assert err_wo <= TOL, err_wo
    # LM head on sampled rows + greedy argmax of the GPU's logits
    lq, ld = synth.q4_blocks(shape.vocab, D, 0, synth.LM_HEAD_ID)
    logits = np_of(dm.logits)
    xf = ref.rmsnorm(np_of(dm.x))
    rows = np.unique(np.concatenate([np.random.default_rng(1).integers(0, shape.vocab, 256),
                                     [int(np.argmax(logits))]]))
    err_lm = gemv_err(logits[rows][None], xf[None], lq[rows], ld[rows])
    assert err_lm <= TOL, err_lm
    assert int(dm.token.item()) == int(np.argmax(logits))
    # end to end (reported, not gated): the oracle's own fp64 layer from x0
    Wd = {k: ref.q4_weights(*v) for k, v in w.items()}
    k0, v0 = synth.decoder_layer_cache(shape, 0, 0, dm.W)
    st = ref.decoder_layer(x0, Wd, k0.copy(), v0.copy(), 1024, shape.n_q_heads, shape.n_kv_heads)
    e2e = np.max(np.abs(np_of(dm.x) - st["out"])) / np.max(np.abs(st["out"]))
    print(f"decoder layer end-to-end max rel error {e2e:.3e}")


def test_decoder_step_full_wrapped(env):
    """The bench's workload: 26 layers, cache filled to 8192 + 300.  Both
    forms of the step run from the same state (the written cache slots, the
    position and the token are restored in between); each is checked kernel
    by kernel on its own inputs, and a second step of each advances the ring."""
    torch, V, WL = env
    shape = synth.DecoderShape()
    filled = 8192 + 300
    dm = WL.DecoderModel(shape, seed=0, filled=filled, token=17)
    slot = filled % dm.W
    saved = [(dm.k_cache[l][:, slot:slot + 2].clone(), dm.v_cache[l][:, slot:slot + 2].clone()) for l in range(dm.L)]
    lq, ld = synth.q4_blocks(shape.vocab, shape.dim, 0, synth.LM_HEAD_ID)
    tokens = {}
    for form in FORMS:
        for l in range(dm.L):
            dm.k_cache[l][:, slot:slot + 2].copy_(saved[l][0])
            dm.v_cache[l][:, slot:slot + 2].copy_(saved[l][1])
        dm.pos.fill_(filled)
        dm.token.fill_(17)
        run_step(dm, form)
        torch.cuda.synchronize()
        assert V.vox_device_status(True) == 0
        assert int(dm.pos.item()) == filled + 1
        check_layer_tail(shape, shape.n_layers - 1, dm, 0, filled)
        logits = np_of(dm.logits)
        xf = ref.rmsnorm(np_of(dm.x))
        rows = np.unique(np.concatenate([np.random.default_rng(2).integers(0, shape.vocab, 512),
                                         [int(np.argmax(logits))]]))
        err_lm = gemv_err(logits[rows][None], xf[None], lq[rows], ld[rows])
        assert err_lm <= TOL, (form, err_lm)
        assert int(dm.token.item()) == int(np.argmax(logits))
        top2 = np.sort(logits)[-2:]
        tokens[form] = (int(dm.token.item()), float(top2[1] - top2[0]), float(np.abs(logits).max()))
        # a second step advances the ring by one slot and reads the new token
        run_step(dm, form)
        torch.cuda.synchronize()
        assert V.vox_device_status(True) == 0
        assert int(dm.pos.item()) == filled + 2
        assert int(dm.token.item()) == int(np.argmax(np_of(dm.logits)))
    # the two forms pick the same token unless the top two logits are within rounding
    (ta, ma, sa), (tb, mb, sb) = tokens["persistent"], tokens["kernels"]
    if min(ma, mb) > 1e-3 * max(sa, sb):
        assert ta == tb, tokens


@pytest.mark.parametrize("form", FORMS)
def test_decoder_step_graph_replay_matches_eager(env, form):
    """The captured step replays exactly what the eager step computes."""
    torch, V, WL = env
    shape = synth.DecoderShape(n_layers=2)
    a = WL.DecoderModel(shape, seed=3, filled=500, token=9)
    b = WL.DecoderModel(shape, seed=3, filled=500, token=9)
    for _ in range(3):
        run_step(a, form)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        run_step(b, form, s)                              # warm-up outside capture
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run_step(b, form)
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    assert V.vox_device_status(True) == 0
    assert int(a.pos.item()) == int(b.pos.item()) == 503
    assert int(a.token.item()) == int(b.token.item())
    assert torch.equal(a.logits, b.logits)
    for l in range(2):
        assert torch.equal(a.k_cache[l].view(torch.int16), b.k_cache[l].view(torch.int16))


SMALL = dict(n_layers=2, dim=256, n_q_heads=4, n_kv_heads=2, head_dim=128, ffn=512, vocab=1024)


@pytest.mark.parametrize("window,filled", [(64, 70), (100, 30), (100, 0), (48, 47), (8192, 8492)])
def test_persistent_step_small_shapes(env, window, filled):
    """A small decoder whose projections have a handful of 16-row tiles, so
    nearly every tile is cut between warps and CTAs; windows that are not a
    multiple of the 16-slot unit, a cache with one valid slot, and a full
    window.  Every kernel of the last layer, the LM head and the argmax are
    checked against the oracle; the per-kernel sequence must agree."""
    torch, V, WL = env
    shape = synth.DecoderShape(window=window, **SMALL)
    out = {}
    for form in FORMS:
        dm = WL.DecoderModel(shape, seed=5, filled=filled, token=3)
        run_step(dm, form)
        torch.cuda.synchronize()
        assert V.vox_device_status(True) == 0
        assert int(dm.pos.item()) == filled + 1
        check_layer_tail(shape, shape.n_layers - 1, dm, 5, filled)
        lq, ld = synth.q4_blocks(shape.vocab, shape.dim, 5, synth.LM_HEAD_ID)
        logits = np_of(dm.logits)
        xf = ref.rmsnorm(np_of(dm.x))
        err = gemv_err(logits[None], xf[None], lq, ld)
        assert err <= TOL, (form, err)
        assert int(dm.token.item()) == int(np.argmax(logits))
        out[form] = np_of(dm.x)
    # the forms reach the same residual stream within the tolerance's scale
    for form in ("persistent", "fused"):
        assert np.max(np.abs(out[form] - out["kernels"])) <= 1e-2 * np.max(np.abs(out["kernels"]))


def test_persistent_step_first_layer_from_embedding(env):
    """The persistent step reads layer 0's input straight from the packed
    embedding table: x after the step's embedding is the exact fp32 row, and
    the first layer's QKV is checked on it."""
    torch, V, WL = env
    shape = synth.DecoderShape(window=64, **dict(SMALL, n_layers=1))
    tok = 777
    dm = WL.DecoderModel(shape, seed=6, filled=10, token=tok)
    run_step(dm, "persistent")
    torch.cuda.synchronize()
    assert V.vox_device_status(True) == 0
    eq, ed = synth.q4_blocks(shape.vocab, shape.dim, 6, synth.EMB_ID)
    x0 = ref.c_dequant_f32(eq, ed, row0=tok, nrows=1)[0]
    # h = x0 + Wo o: the residual used the embedding row exactly
    w = synth.decoder_layer_weights(shape, 0, 6)
    err_wo = gemv_err((np_of(dm.h) - x0)[None], np_of(dm.attn)[None], *w["wo"])
    assert err_wo <= TOL, err_wo
    qs = np.concatenate([w["wq"][0], w["wk"][0], w["wv"][0]])
    ds = np.concatenate([w["wq"][1], w["wk"][1], w["wv"][1]])
    err_qkv = gemv_err(np_of(dm.qkv)[None], ref.rmsnorm(x0)[None], qs, ds)
    assert err_qkv <= TOL, err_qkv


def check_encoder_layer(shape, em, layer, seed):
    """Every kernel of encoder layer `layer` on the GPU's own inputs to it:
    the tap holds the layer's input x and its residual h after attention; the
    qkv / att / up buffers and x hold that layer's values after the call."""
    D, F, R, nh, hd = shape.dim, shape.ffn, shape.rows, shape.n_heads, shape.head_dim
    w = synth.encoder_layer_weights(shape, layer, seed)
    tap = np_of(em.tap).astype(np.float64)
    x_in, h = tap[0], tap[1]
    qkv_b = bits(em.qkv)
    # QKV GEMM on bf16(RMSNorm(x_in)); the output is stored as bf16
    xn = ref.bf16_to_f64(ref.f32_to_bf16(ref.rmsnorm(x_in).astype(np.float32)))
    err = gemv_err(ref.bf16_to_f64(qkv_b), xn, *w["wqkv"])
    assert err <= TOL, ("qkv", err)
    # window attention on the GPU's q, k, v and the history
    kh, vh = synth.encoder_layer_history(shape, layer, seed)
    Q = ref.bf16_to_f64(qkv_b[:, :D])
    K = np.concatenate([ref.bf16_to_f64(kh), ref.bf16_to_f64(qkv_b[:, D:2 * D])])
    Vv = np.concatenate([ref.bf16_to_f64(vh), ref.bf16_to_f64(qkv_b[:, 2 * D:])])
    rows = list(range(0, R, 15)) + [R - 1]
    att_ref = np.concatenate([ref.window_attn(Q[i:i + 1], K, Vv, shape.window + i, shape.window, nh, hd)
                              for i in rows])
    att = ref.bf16_to_f64(bits(em.att))
    # the chunk stores the attention output as bf16 (the O GEMM's operand
    # type): half a bf16 ulp of the stored value is the format's own share
    half_ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(att_ref), 1e-30))) - 8)
    for ii, i in enumerate(rows):
        p = shape.window + i
        lo = p - shape.window + 1
        for hh in range(nh):
            sl = slice(hh * hd, (hh + 1) * hd)
            sc = (K[lo:p + 1, sl] @ Q[i, sl]) / math.sqrt(hd)
            pr = np.exp(sc - sc.max()); pr /= pr.sum()
            den = np.linalg.norm(pr) * np.linalg.norm(Vv[lo:p + 1, sl], axis=0)
            excess = np.maximum(np.abs(att[i, sl] - att_ref[ii, sl]) - half_ulp[ii, sl], 0.0)
            assert np.max(excess / den) <= TOL, ("attention", i, hh)
    # O GEMM + residual: h = x_in + Wo att
    err_o = gemv_err(h - x_in, att, *w["wo"])
    assert err_o <= TOL, ("o", err_o)
    # up GEMM + GELU on bf16(RMSNorm(h)), stored as bf16
    up = ref.bf16_to_f64(bits(em.up))
    n2 = ref.bf16_to_f64(ref.f32_to_bf16(ref.rmsnorm(h).astype(np.float32)))
    Wup = ref.q4_weights(*w["wup"])
    err_up = ref.gemv_error(up, ref.gelu(n2 @ Wup.T), n2, Wup)
    assert err_up <= TOL, ("up", err_up)
    # down GEMM + residual: x_out = h + Wdown up
    x_out = np_of(em.x).astype(np.float64)
    err_dn = gemv_err(x_out - h, up, *w["wdown"])
    assert err_dn <= TOL, ("down", err_dn)
    return x_out


def test_encoder_layer_and_adapter(env):
    torch, V, WL = env
    shape = synth.EncoderShape()
    em = WL.EncoderModel(shape, seed=0, n_layers=1, tap=True)
    em.run()
    torch.cuda.synchronize()
    assert V.vox_device_status(True) == 0
    D, R = shape.dim, shape.rows
    x0 = synth.activations(R, D, 0, synth.ENC_X_ID)
    assert np.array_equal(np_of(em.tap[0]), x0)                 # layer 0's input is the chunk input
    x1 = check_encoder_layer(shape, em, 0, 0)
    check_adapter(shape, em, x1, 0)


def check_adapter(shape, em, x_out, seed):
    """The adapter on the downsampled bf16 rows of the chunk output: the first
    Linear + GELU (stored as bf16) on the GPU's input, the second Linear on the
    GPU's GELU output; the oracle's whole adapter is reported."""
    aq, ad = synth.q4_blocks(shape.adapter_out, 4 * shape.dim, seed, synth.ADAPTER_ID)
    a2q, a2d = synth.q4_blocks(shape.adapter_out, shape.adapter_out, seed, synth.ADAPTER2_ID)
    xd = ref.downsample_rows(ref.bf16_to_f64(ref.f32_to_bf16(x_out.astype(np.float32))), 4)
    W1 = ref.q4_weights(aq, ad)
    mid = ref.bf16_to_f64(bits(em.mid))
    err1 = ref.gemv_error(mid, ref.gelu(xd @ W1.T), xd, W1)
    assert err1 <= TOL, ("adapter linear 1 + gelu", err1)
    err2 = gemv_err(np_of(em.out), mid, a2q, a2d)
    assert err2 <= TOL, ("adapter linear 2", err2)
    full = ref.adapter(xd, W1, ref.q4_weights(a2q, a2d))
    e2e = np.max(np.abs(np_of(em.out) - full)) / np.max(np.abs(full))
    print(f"adapter end-to-end max rel error {e2e:.3e}")


def test_encoder_chunk_last_layer(env):
    """The full 32-layer chunk that the bench times: its last layer checked
    kernel by kernel on that layer's own GPU inputs, and the adapter."""
    torch, V, WL = env
    shape = synth.EncoderShape()
    em = WL.EncoderModel(shape, seed=0, tap=True)
    em.run()
    torch.cuda.synchronize()
    assert V.vox_device_status(True) == 0
    x_out = check_encoder_layer(shape, em, shape.n_layers - 1, 0)
    assert np.all(np.isfinite(x_out))
    check_adapter(shape, em, x_out, 0)


@pytest.mark.parametrize("form", FORMS)
def test_decoder_layer_rope(env, form):
    """One layer with the rotary embedding on (theta 1e6) at position 1024,
    both forms: q and k turned back by the oracle's inverse rotation match
    the plain QKV product, the cache holds the rotated k, and the rest of the
    layer is checked on the GPU's own inputs."""
    torch, V, WL = env
    shape = synth.DecoderShape()
    tok, theta, filled = 4242, 1e6, 1024
    dm = WL.DecoderModel(shape, seed=0, n_layers=1, filled=filled, token=tok, rope_theta=theta)
    run_step(dm, form)
    torch.cuda.synchronize()
    assert V.vox_device_status(True) == 0
    D, QD, KVD, hd = shape.dim, shape.q_dim, shape.kv_dim, shape.head_dim
    eq, ed = synth.q4_blocks(shape.vocab, D, 0, synth.EMB_ID)
    x0 = ref.c_dequant_f32(eq, ed, row0=tok, nrows=1)[0]
    w = synth.decoder_layer_weights(shape, 0, 0)
    qs = np.concatenate([w["wq"][0], w["wk"][0], w["wv"][0]])
    ds = np.concatenate([w["wq"][1], w["wk"][1], w["wv"][1]])
    qkv = np_of(dm.qkv).astype(np.float64)
    back = qkv.copy()
    back[:QD] = ref.rope(qkv[:QD], -filled, theta, hd)
    back[QD:QD + KVD] = ref.rope(qkv[QD:QD + KVD], -filled, theta, hd)
    err = gemv_err(back[None], ref.rmsnorm(x0)[None], qs, ds)
    assert err <= TOL, err
    check_layer_tail(shape, 0, dm, 0, filled)


def test_encoder_streaming_two_chunks(env):
    """Two chunks streamed through a 1-layer encoder: after the first, the
    next history is bit for bit the oracle's roll of the old history and the
    chunk's own k, v rows; the second chunk's window attention, on the GPU's
    q, k, v and that history, matches the oracle."""
    torch, V, WL = env
    shape = synth.EncoderShape(n_layers=1)
    D, R, W, nh, hd = shape.dim, shape.rows, shape.window, shape.n_heads, shape.head_dim
    em = WL.EncoderModel(shape, seed=0, n_layers=1, stream=True)
    kh0, vh0 = bits(em.k_hist[0]), bits(em.v_hist[0])
    em.reset()
    em.run()
    torch.cuda.synchronize()
    assert V.vox_device_status(True) == 0
    qkv1 = bits(em.qkv)
    assert np.array_equal(bits(em.k_next[0]), ref.roll_history(kh0, qkv1[:, D:2 * D], W))
    assert np.array_equal(bits(em.v_next[0]), ref.roll_history(vh0, qkv1[:, 2 * D:], W))
    em.swap_history()
    em.set_input(synth.activations(R, D, 0, synth.ENC_X_ID + 7))
    em.run()
    torch.cuda.synchronize()
    assert V.vox_device_status(True) == 0
    kh, vh = bits(em.k_hist[0]), bits(em.v_hist[0])
    qkv = bits(em.qkv)
    Q = ref.bf16_to_f64(qkv[:, :D])
    K = np.concatenate([ref.bf16_to_f64(kh), ref.bf16_to_f64(qkv[:, D:2 * D])])
    Vv = np.concatenate([ref.bf16_to_f64(vh), ref.bf16_to_f64(qkv[:, 2 * D:])])
    att = ref.bf16_to_f64(bits(em.att))
    for i in list(range(0, R, 17)) + [R - 1]:
        o_ref = ref.window_attn(Q[i:i + 1], K, Vv, W + i, W, nh, hd)[0]
        p = W + i
        half_ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(o_ref), 1e-30))) - 8)
        for hh in range(nh):
            sl = slice(hh * hd, (hh + 1) * hd)
            sc = (K[p - W + 1:p + 1, sl] @ Q[i, sl]) / math.sqrt(hd)
            pr = np.exp(sc - sc.max()); pr /= pr.sum()
            den = np.linalg.norm(pr) * np.linalg.norm(Vv[p - W + 1:p + 1, sl], axis=0)
            excess = np.maximum(np.abs(att[i, sl] - o_ref[sl]) - half_ulp[sl], 0.0)
            assert np.max(excess / den) <= TOL, ("attention", i, hh)
