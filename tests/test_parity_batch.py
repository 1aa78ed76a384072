"""Parity of the batched decode path with the oracle: several sequences, each
with its own rolling cache in 64-slot pages of shared pools.

* vox_gqa_decode_attn_paged against the oracle's single-sequence attention on
  each sequence's gathered cache (pages in a random order, positions from 0
  to past a wrap, never-written slots filled with NaN bits);
* the VOX_EP_KV_APPEND_PAGED epilogue of the GEMV: the new k, v rows land
  bit for bit in the page and row the table names, and nowhere else;
* vox_decoder_batch_step, kernel by kernel on the GPU's own inputs for every
  sequence (teacher forcing), plus a CUDA-graph replay that matches eager.
Tolerance: the oracle module's normalised error <= 2e-3; cache bits exact.
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


def status(V):
    import torch

    torch.cuda.synchronize()
    return V.vox_device_status(True)


def nan_unwritten(pool, table, positions, W):
    """Slots a sequence has not written yet hold NaN bits (they must not be read)."""
    pool = pool.copy()
    for s, pos in enumerate(positions):
        nv = min(pos + 1, W)
        for slot in range(nv, W):
            pool[table[s][slot // ref.PAGE_SLOTS], :, slot % ref.PAGE_SLOTS, :] = 0x7FC1
    return pool


def paged_case(env, n_q, n_kv, W, positions, seed=0, nan_fill=True, spare=3, bad_page=None):
    torch, V, WL = env
    hd = 128
    n_seq = len(positions)
    shape = synth.DecoderShape(n_layers=1, n_q_heads=n_q, n_kv_heads=n_kv, head_dim=hd, window=W)
    n_pages = n_seq * (W // ref.PAGE_SLOTS) + spare
    kb, vb = synth.page_pool(shape, 0, n_pages, seed)
    table = synth.page_table(n_seq, W, n_pages, seed)
    if nan_fill:
        kb, vb = nan_unwritten(kb, table, positions, W), nan_unwritten(vb, table, positions, W)
    table_dev = table.copy()
    if bad_page is not None:
        s, c = bad_page
        table_dev[s, c] = n_pages + 5
    q = synth.activations(n_seq * n_q, hd, seed, 13).reshape(n_seq, n_q, hd) * 2.0
    out = torch.full((n_seq, n_q, hd), float("nan"), device="cuda")
    wsb = V.vox_gqa_decode_attn_paged_workspace(n_seq, n_q, n_kv, hd, W)
    ws = torch.full((wsb,), 0xFF, dtype=torch.uint8, device="cuda")    # no initial contents needed
    V.vox_gqa_decode_attn_paged(WL.to_dev(q, "cuda"), WL.bf16_dev(kb, "cuda"), WL.bf16_dev(vb, "cuda"), n_pages,
                                WL.to_dev(table_dev, "cuda"),
                                torch.tensor(positions, dtype=torch.int64, device="cuda"), n_seq, out, n_q, n_kv,
                                hd, W, 1.0 / math.sqrt(hd), ws, wsb)
    st = status(V)
    o = np_of(out)
    errs = []
    for s, pos in enumerate(positions):
        kc, vc = ref.paged_to_cache(kb, table[s]), ref.paged_to_cache(vb, table[s])
        o_ref = ref.c_gqa_attn(q[s], kc, vc, pos)
        nv = min(pos + 1, W)
        errs.append(ref.attn_error(o[s], o_ref, ref.attn_probs(q[s], kc, pos), ref.bf16_to_f64(vc[:, :nv]),
                                   n_q // n_kv))
    return st, errs, o


@pytest.mark.parametrize("n_q,n_kv,W,positions", [
    (32, 8, 512, [100, 300 + 2 * 512, 0]),
    (32, 8, 8192, [8491, 100, 8192 + 5, 64, 63, 0, 4000, 3 * 8192 + 17]),
    (4, 1, 64, [70]),
    (16, 2, 192, [191, 192, 1, 130, 64]),
])
def test_paged_attention(env, n_q, n_kv, W, positions):
    st, errs, o = paged_case(env, n_q, n_kv, W, positions)
    assert st == 0
    assert np.all(np.isfinite(o))
    assert max(errs) <= TOL, errs


def test_paged_attention_page_outside_pool(env):
    """A table entry past the pool reads zeros for that chunk and sets the
    status word; the other sequences are unaffected."""
    st, errs, o = paged_case(env, 32, 8, 256, [255, 100], bad_page=(0, 1))
    assert st == 0x203
    assert errs[1] <= TOL, errs


def test_gemv_kv_append_paged(env):
    """m = 3 sequences through the QKV GEMV with the paged append: y within
    tolerance, each sequence's k, v in bf16 at its slot's page and row, and
    every other pool element unchanged."""
    torch, V, WL = env
    n_q, n_kv, hd, W, k = 4, 2, 128, 128, 256
    QD, KVD = n_q * hd, n_kv * hd
    n = QD + 2 * KVD
    positions = [5, 64 + 3, 2 * W + 127]
    m = len(positions)
    qs, d = synth.q4_blocks(n, k, 0, 8100)
    packed, w = WL.pack_q4(qs, d, "cuda")
    x = synth.activations(m, k, 0, 8101)
    shape = synth.DecoderShape(n_layers=1, n_q_heads=n_q, n_kv_heads=n_kv, head_dim=hd, window=W)
    n_pages = m * (W // ref.PAGE_SLOTS) + 2
    kb, vb = synth.page_pool(shape, 0, n_pages, 8102)
    table = synth.page_table(m, W, n_pages, 8103)
    kp, vp = WL.bf16_dev(kb, "cuda"), WL.bf16_dev(vb, "cuda")
    tdev = WL.to_dev(table, "cuda")
    pdev = torch.tensor(positions, dtype=torch.int64, device="cuda")
    y = torch.full((m, n), float("nan"), device="cuda")
    e = V.vox_epilogue(op=V.VOX_EP_KV_APPEND_PAGED, k_cache=kp.data_ptr(), v_cache=vp.data_ptr(), n_kv_heads=n_kv,
                       head_dim=hd, window=W, q_rows=QD, pos_dev=pdev.data_ptr(), page_table=tdev.data_ptr(),
                       n_pages=n_pages)
    wsb = V.vox_q4_gemv_workspace(w, m, e)
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    V.vox_q4_gemv(w, WL.to_dev(x, "cuda"), m, k, y, n, e, ws, wsb)
    assert status(V) == 0
    yv = np_of(y)
    W_ = ref.q4_weights(qs, d)
    assert ref.gemv_error(yv, x.astype(np.float64) @ W_.T, x, W_) <= TOL
    kw, vw = kb.copy(), vb.copy()
    for s, pos in enumerate(positions):
        ref.paged_append(kw, vw, table[s], yv[s, QD:QD + KVD].reshape(n_kv, hd), yv[s, QD + KVD:].reshape(n_kv, hd),
                         pos)
    assert np.array_equal(bits(kp), kw) and np.array_equal(bits(vp), vw)
    assert not np.array_equal(kw, kb)


def batch_shape():
    return synth.DecoderShape(n_layers=1)


def check_batch_layer(shape, bm, seq, positions, tokens, seed=0):
    """Every kernel of the (single) layer and the LM head for sequence `seq`,
    on the GPU's own inputs."""
    D, QD, KVD, F = shape.dim, shape.q_dim, shape.kv_dim, shape.ffn
    pos = positions[seq]
    w = synth.decoder_layer_weights(shape, 0, seed)
    # x0 = embedding row of the token, exact
    eq, ed = synth.q4_blocks(shape.vocab, D, seed, synth.EMB_ID)
    x0 = ref.c_dequant_f32(eq, ed, row0=tokens[seq], nrows=1)[0]
    qkv = np_of(bm.qkv)[seq]
    qs = np.concatenate([w["wq"][0], w["wk"][0], w["wv"][0]])
    ds = np.concatenate([w["wq"][1], w["wk"][1], w["wv"][1]])
    Wqkv = ref.q4_weights(qs, ds)
    n0 = ref.rmsnorm(x0)
    assert ref.gemv_error(qkv[None], (n0 @ Wqkv.T)[None], n0, Wqkv) <= TOL
    # the paged append: the sequence's slot, in its page, holds bf16 of k and v
    kp, vp = bits(bm.k_pool[0]), bits(bm.v_pool[0])
    table = bm.table_np[seq]
    slot = pos % bm.W
    page, row = table[slot // ref.PAGE_SLOTS], slot % ref.PAGE_SLOTS
    assert np.array_equal(kp[page, :, row], ref.f32_to_bf16(qkv[QD:QD + KVD]).reshape(shape.n_kv_heads, -1))
    assert np.array_equal(vp[page, :, row], ref.f32_to_bf16(qkv[QD + KVD:]).reshape(shape.n_kv_heads, -1))
    # attention on the GPU's q and the sequence's gathered cache
    kc, vc = ref.paged_to_cache(kp, table), ref.paged_to_cache(vp, table)
    q = qkv[:QD].reshape(shape.n_q_heads, shape.head_dim)
    o = np_of(bm.attn)[seq].reshape(shape.n_q_heads, shape.head_dim)
    nv = min(pos + 1, bm.W)
    err = ref.attn_error(o, ref.c_gqa_attn(q, kc, vc, pos), ref.attn_probs(q, kc, pos), ref.bf16_to_f64(vc[:, :nv]),
                         shape.n_q_heads // shape.n_kv_heads)
    assert err <= TOL, err
    # Wo + residual, W1||W3 + SiLU*mul, W2 + residual on the GPU's inputs
    h = np_of(bm.h)[seq]
    Wo = ref.q4_weights(*w["wo"])
    attn = np_of(bm.attn)[seq]
    assert ref.gemv_error((h - x0)[None], (attn @ Wo.T)[None], attn, Wo) <= TOL
    n2 = ref.rmsnorm(h)
    W1, W3 = ref.q4_weights(*w["w1"]), ref.q4_weights(*w["w3"])
    g, u = n2 @ W1.T, n2 @ W3.T
    a = np_of(bm.act)[seq]
    bound = 1.1 * np.abs(u) * np.linalg.norm(n2) * np.linalg.norm(W1, axis=1) + \
        np.abs(ref.silu(g)) * np.linalg.norm(n2) * np.linalg.norm(W3, axis=1)
    assert np.all(np.abs(a - ref.silu(g) * u) <= TOL * bound)
    W2 = ref.q4_weights(*w["w2"])
    xo = np_of(bm.x)[seq]
    assert ref.gemv_error((xo - h)[None], (a @ W2.T)[None], a, W2) <= TOL
    # LM head on sampled rows and the greedy token
    lq, ld = synth.q4_blocks(shape.vocab, D, seed, synth.LM_HEAD_ID)
    logits = np_of(bm.logits)[seq]
    xf = ref.rmsnorm(xo)
    rows = np.unique(np.concatenate([np.random.default_rng(3 + seq).integers(0, shape.vocab, 256),
                                     [int(np.argmax(logits))]]))
    Wl = ref.q4_weights(lq[rows], ld[rows])
    assert ref.gemv_error(logits[rows][None], (xf @ Wl.T)[None], xf, Wl) <= TOL
    return int(np.argmax(logits))


@pytest.mark.parametrize("positions,tokens", [
    # 3 sequences: every projection on the multi-row GEMV
    ([1024, 8192 + 300, 0], [17, 4242, 131071]),
    # from 4 sequences on Wo and W2 run on the tcgen05 GEMM over bf16 inputs
    ([1024, 8192 + 300, 0, 64], [17, 4242, 131071, 9]),
    ([1024, 8192 + 300, 0, 64, 63, 5000, 8191], [17, 4242, 131071, 9, 0, 77, 65536]),
])
def test_batch_step_one_layer(env, positions, tokens):
    """Three, four or seven sequences at different positions (fresh, mid,
    wrapped, first and last slot of a page): every kernel checked per sequence,
    positions advanced, tokens = per-row argmax; a second step writes the
    next slots."""
    torch, V, WL = env
    shape = batch_shape()
    bm = WL.BatchDecoderModel(shape, len(positions), positions, tokens, n_layers=1)
    bm.step()
    assert status(V) == 0
    assert np_of(bm.pos).tolist() == [p + 1 for p in positions]
    new_tokens = np_of(bm.token).tolist()
    for s in range(len(positions)):
        assert new_tokens[s] == check_batch_layer(shape, bm, s, positions, tokens)
    bm.step()
    assert status(V) == 0
    assert np_of(bm.pos).tolist() == [p + 2 for p in positions]
    for s in range(len(positions)):
        assert check_batch_layer(shape, bm, s, [p + 1 for p in positions], new_tokens) == int(np_of(bm.token)[s])


def test_batch_step_graph_replay_matches_eager(env):
    torch, V, WL = env
    shape = synth.DecoderShape(n_layers=2)
    positions = [300, 8192 + 1, 5]
    tokens = [1, 2, 3]
    bm = WL.BatchDecoderModel(shape, 3, positions, tokens, n_layers=2)
    saved = [(bm.k_pool[l].clone(), bm.v_pool[l].clone()) for l in range(2)]

    def reset():
        for l in range(2):
            bm.k_pool[l].copy_(saved[l][0])
            bm.v_pool[l].copy_(saved[l][1])
        bm.pos.copy_(torch.tensor(positions, dtype=torch.int64))
        bm.token.copy_(torch.tensor(tokens, dtype=torch.int32))

    bm.step()
    assert status(V) == 0
    eager = (np_of(bm.logits).copy(), np_of(bm.token).copy())
    g = bm.capture()
    reset()
    g.replay()
    assert status(V) == 0
    assert np.array_equal(np_of(bm.logits), eager[0]) and np.array_equal(np_of(bm.token), eager[1])
    assert np_of(bm.pos).tolist() == [p + 1 for p in positions]
    del g
