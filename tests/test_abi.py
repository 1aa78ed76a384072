"""The C ABI: libvox.so loads without a GPU, exports every entry point that
include/vox.h declares, and rejects bad arguments on the host with the
documented status codes before launching anything."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "vox.h")


@pytest.fixture(scope="module")
def V():
    from bit_quantized_transformer_b200 import build

    build.build()
    from bit_quantized_transformer_b200 import vox

    return vox


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(vox_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("vox_q4_dequant", "vox_q4_gemv", "vox_q4_gemm", "vox_kv_append_rolling", "vox_gqa_decode_attn",
                 "vox_q4_pack", "vox_decoder_step", "vox_encoder_chunk"):
        assert must in names


def test_library_exports_every_declared_symbol(V):
    missing = [n for n in declared_functions() if not hasattr(V.lib, n)]
    assert not missing, missing


def test_library_exports_nothing_undeclared(V):
    import subprocess

    out = subprocess.run(["nm", "-D", "--defined-only", V.LIB_PATH], capture_output=True, text=True).stdout
    exported = sorted({l.split()[-1] for l in out.splitlines() if " T vox_" in l})
    assert exported == declared_functions()


def test_status_strings(V):
    assert V.lib.vox_status_str(0) == b"VOX_OK"
    assert V.lib.vox_status_str(V.VOX_ERR_WORKSPACE) == b"VOX_ERR_WORKSPACE"
    assert V.lib.vox_status_str(99) == b"VOX_ERR_UNKNOWN"


def test_packed_bytes(V):
    assert V.vox_q4_packed_bytes(4096, 3072) == 4096 * 3072 * 18 // 32
    assert V.vox_q4_packed_bytes(17, 32) == 32 * 64 * 18 // 32        # padded to 2 tiles x 1 chunk
    assert V.vox_q4_packed_bytes(16, 48) == -1
    assert V.vox_q4_packed_bytes(0, 64) == -1


FAKE = 0x10000          # a 16-byte aligned address; never dereferenced: validation fails first


def test_pack_validation(V):
    L = V.lib
    assert L.vox_q4_pack(None, 16, 64, 0, FAKE, None) == V.VOX_ERR_NULL
    assert L.vox_q4_pack(FAKE, 16, 48, 0, FAKE, None) == V.VOX_ERR_SHAPE
    assert L.vox_q4_pack(FAKE, 0, 64, 0, FAKE, None) == V.VOX_ERR_SHAPE
    assert L.vox_q4_pack(FAKE, 16, 64, 7, FAKE, None) == V.VOX_ERR_RANGE
    assert L.vox_q4_pack(FAKE, 24, 64, V.VOX_PACK_GATE_UP, FAKE, None) == V.VOX_ERR_SHAPE
    assert L.vox_q4_pack(FAKE, 16, 64, 0, FAKE + 4, None) == V.VOX_ERR_ALIGN


def test_dequant_validation(V):
    L = V.lib
    w = V.vox_q4_weight(FAKE, 32, 64)
    assert L.vox_q4_dequant(ctypes.byref(w), 0, 1, None, V.VOX_F32, 64, None) == V.VOX_ERR_NULL
    assert L.vox_q4_dequant(ctypes.byref(w), 0, 1, FAKE, V.VOX_F16, 64, None) == V.VOX_ERR_DTYPE
    assert L.vox_q4_dequant(ctypes.byref(w), 31, 2, FAKE, V.VOX_F32, 64, None) == V.VOX_ERR_RANGE
    assert L.vox_q4_dequant(ctypes.byref(w), -1, 1, FAKE, V.VOX_F32, 64, None) == V.VOX_ERR_RANGE
    assert L.vox_q4_dequant(ctypes.byref(w), 0, 1, FAKE, V.VOX_F32, 63, None) == V.VOX_ERR_SHAPE
    bad = V.vox_q4_weight(FAKE + 8, 32, 64)
    assert L.vox_q4_dequant(ctypes.byref(bad), 0, 1, FAKE, V.VOX_F32, 64, None) == V.VOX_ERR_ALIGN
    assert L.vox_q4_dequant(None, 0, 1, FAKE, V.VOX_F32, 64, None) == V.VOX_ERR_NULL


def test_gemv_validation(V):
    L = V.lib
    w = V.vox_q4_weight(FAKE, 64, 96)
    ws = V.vox_q4_gemv_workspace(w, 1, None)
    assert ws > 0
    g = lambda m=1, ldx=96, ldy=64, ep=None, wsp=FAKE, wsb=ws, x=FAKE, y=FAKE: L.vox_q4_gemv(
        ctypes.byref(w), x, m, ldx, y, ldy, ctypes.byref(ep) if ep else None, wsp, wsb, None)
    assert g(x=None) == V.VOX_ERR_NULL
    assert g(m=0) == V.VOX_ERR_SHAPE
    assert g(m=9) == V.VOX_ERR_SHAPE
    assert g(ldx=95) == V.VOX_ERR_SHAPE
    assert g(ldy=63) == V.VOX_ERR_SHAPE
    assert g(wsp=None) == V.VOX_ERR_WORKSPACE
    assert g(wsb=ws - 1) == V.VOX_ERR_WORKSPACE
    ep = V.vox_epilogue(op=V.VOX_EP_RESIDUAL, residual=None, ldr=64)
    assert g(ep=ep) == V.VOX_ERR_NULL
    ep = V.vox_epilogue(op=9)
    assert g(ep=ep) == V.VOX_ERR_RANGE
    ep = V.vox_epilogue(op=V.VOX_EP_KV_APPEND, k_cache=FAKE, v_cache=FAKE, n_kv_heads=1, head_dim=32, window=4,
                        q_rows=8, pos=0)
    assert g(ep=ep) == V.VOX_ERR_SHAPE            # 8 + 2*32 rows > 64
    ep = V.vox_epilogue(op=V.VOX_EP_KV_APPEND, k_cache=FAKE, v_cache=FAKE, n_kv_heads=1, head_dim=16, window=4,
                        q_rows=8, pos=-1)
    assert g(ep=ep) == V.VOX_ERR_RANGE
    ep = V.vox_epilogue(op=V.VOX_EP_ARGMAX, argmax=None)
    assert g(ep=ep) == V.VOX_ERR_NULL
    wide = V.vox_q4_weight(FAKE, 64, 16384)
    assert L.vox_q4_gemv(ctypes.byref(wide), FAKE, 8, 16384, FAKE, 64, None, FAKE, 1 << 30, None) == V.VOX_ERR_SHAPE
    ep = V.vox_epilogue(op=V.VOX_EP_SILU_MUL)
    w24 = V.vox_q4_weight(FAKE, 24, 96)
    assert L.vox_q4_gemv(ctypes.byref(w24), FAKE, 1, 96, FAKE, 24, ctypes.byref(ep), FAKE, 1 << 30,
                         None) == V.VOX_ERR_SHAPE


def test_gemm_validation(V):
    L = V.lib
    w = V.vox_q4_weight(FAKE, 128, 128)
    g = lambda xd=V.VOX_BF16, m=16, ldx=128, yd=V.VOX_F32, ldy=128, ep=None, x=FAKE: L.vox_q4_gemm(
        ctypes.byref(w), x, xd, m, ldx, FAKE, yd, ldy, ctypes.byref(ep) if ep else None, None)
    assert g(x=None) == V.VOX_ERR_NULL
    assert g(xd=V.VOX_F32) == V.VOX_ERR_DTYPE
    assert g(yd=V.VOX_F16) == V.VOX_ERR_DTYPE
    assert g(m=0) == V.VOX_ERR_SHAPE
    assert g(ldx=130) == V.VOX_ERR_SHAPE
    assert g(x=FAKE + 2) == V.VOX_ERR_ALIGN
    assert g(ep=V.vox_epilogue(op=V.VOX_EP_ARGMAX, argmax=FAKE)) == V.VOX_ERR_RANGE
    assert g(ep=V.vox_epilogue(op=V.VOX_EP_RESIDUAL, residual=FAKE, ldr=128), yd=V.VOX_BF16) == V.VOX_ERR_DTYPE
    w96 = V.vox_q4_weight(FAKE, 128, 96)
    assert L.vox_q4_gemm(ctypes.byref(w96), FAKE, V.VOX_BF16, 16, 96, FAKE, V.VOX_F32, 128, None,
                         None) == V.VOX_ERR_SHAPE


def test_matmul_validation(V):
    """vox_q4_matmul checks the GEMM side's arguments on the host (m > 8);
    m <= 8 takes the GEMV's checks."""
    L = V.lib
    w = V.vox_q4_weight(FAKE, 128, 128)
    ws = V.vox_q4_matmul_workspace(w, 16, None)
    assert ws >= 256 + 16 * 128 * 2
    assert V.vox_q4_matmul_workspace(w, 8, None) == V.vox_q4_gemv_workspace(w, 8, None)
    mm = lambda m=16, ldx=128, ep=None, wsp=FAKE, wsb=ws, x=FAKE: L.vox_q4_matmul(
        ctypes.byref(w), x, m, ldx, FAKE, 128, ctypes.byref(ep) if ep else None, wsp, wsb, None)
    assert mm(x=None) == V.VOX_ERR_NULL
    assert mm(m=0) == V.VOX_ERR_SHAPE
    assert mm(ldx=100) == V.VOX_ERR_SHAPE
    assert mm(wsp=None) == V.VOX_ERR_WORKSPACE
    assert mm(wsb=ws - 16) == V.VOX_ERR_WORKSPACE
    assert mm(wsp=FAKE + 8) == V.VOX_ERR_ALIGN
    assert mm(ep=V.vox_epilogue(op=V.VOX_EP_SILU_MUL)) == V.VOX_ERR_RANGE
    assert mm(ep=V.vox_epilogue(op=V.VOX_EP_ARGMAX, argmax=FAKE)) == V.VOX_ERR_RANGE
    assert mm(ep=V.vox_epilogue(op=V.VOX_EP_GELU, rmsnorm=1, eps=-1.0)) == V.VOX_ERR_RANGE
    assert mm(m=4, x=None) == V.VOX_ERR_NULL            # the GEMV's own checks
    w96 = V.vox_q4_weight(FAKE, 128, 96)
    assert L.vox_q4_matmul(ctypes.byref(w96), FAKE, 16, 96, FAKE, 128, None, FAKE, ws, None) == V.VOX_ERR_SHAPE


def test_kv_and_attention_validation(V):
    L = V.lib
    assert L.vox_kv_append_rolling(None, FAKE, FAKE, FAKE, 0, 8, 128, 16, 0, None) == V.VOX_ERR_NULL
    assert L.vox_kv_append_rolling(FAKE, FAKE, FAKE, FAKE, 0, 8, 128, 16, -1, None) == V.VOX_ERR_RANGE
    assert L.vox_kv_append_rolling(FAKE, FAKE, FAKE, FAKE, 0, 8, 128, 0, 0, None) == V.VOX_ERR_RANGE
    assert L.vox_kv_append_rolling(FAKE, FAKE, FAKE, FAKE, 2, 8, 128, 16, 0, None) == V.VOX_ERR_DTYPE
    ws = V.vox_gqa_decode_attn_workspace(32, 8, 128, 8192)
    assert ws > 0
    a = lambda nq=32, nkv=8, hd=128, W=8192, pos=0, wsp=FAKE, wsb=ws, kc=FAKE: L.vox_gqa_decode_attn(
        FAKE, kc, FAKE, FAKE, nq, nkv, hd, W, pos, 0.088, wsp, wsb, None)
    assert a(kc=None) == V.VOX_ERR_NULL
    assert a(nq=30) == V.VOX_ERR_RANGE
    assert a(nq=80, nkv=8) == V.VOX_ERR_RANGE     # group of 10 > 8
    assert a(pos=-1) == V.VOX_ERR_RANGE
    assert a(W=0) == V.VOX_ERR_RANGE
    assert a(hd=64) == V.VOX_ERR_SHAPE
    assert a(wsp=None) == V.VOX_ERR_WORKSPACE
    assert a(wsb=ws - 16) == V.VOX_ERR_WORKSPACE
    assert a(kc=FAKE + 2) == V.VOX_ERR_ALIGN
    assert L.vox_gqa_decode_attn(FAKE, FAKE, FAKE, FAKE + 4, 32, 8, 128, 8192, 0, 0.088, FAKE, ws,
                                 None) == V.VOX_ERR_ALIGN
    assert L.vox_gqa_decode_attn(FAKE, FAKE, FAKE, FAKE + 8, 32, 8, 128, 8192, 0, 0.088, FAKE, ws,
                                 None) == V.VOX_ERR_ALIGN


def test_static_attention_validation(V):
    """The no-workspace entry point rejects bad arguments, and shapes its
    fixed scratch cannot hold, on the host (no device call happens first)."""
    L = V.lib
    s = lambda nq=32, nkv=8, hd=128, W=8192, pos=0, kc=FAKE: L.vox_gqa_decode_attn_static(
        FAKE, kc, FAKE, FAKE, nq, nkv, hd, W, pos, 0.088, None)
    assert s(kc=None) == V.VOX_ERR_NULL
    assert s(nq=30) == V.VOX_ERR_RANGE
    assert s(pos=-1) == V.VOX_ERR_RANGE
    assert s(W=0) == V.VOX_ERR_RANGE
    assert s(hd=64) == V.VOX_ERR_SHAPE
    assert s(kc=FAKE + 2) == V.VOX_ERR_ALIGN
    for off in (4, 8):                                  # out is written with 16-byte stores
        assert L.vox_gqa_decode_attn_static(FAKE, FAKE, FAKE, FAKE + off, 32, 8, 128, 8192, 0, 0.088,
                                            None) == V.VOX_ERR_ALIGN
    assert s(nq=64, nkv=16) == V.VOX_ERR_RANGE          # more kv heads than the scratch holds
    assert b"static scratch" in L.vox_last_error()
    assert s(nq=64, nkv=8) == V.VOX_ERR_RANGE           # groups of 8 > 4
    # seven kv heads pass the head / group limits and stop at the alignment
    # check, still before any device call (the scratch size itself is checked
    # on the GPU by the static-scratch test)
    assert s(nq=28, nkv=7, kc=FAKE + 2) == V.VOX_ERR_ALIGN


def test_window_attn_and_rmsnorm_validation(V):
    L = V.lib
    w = lambda hd=40, W=750, nq=256, ldq=3840, od=V.VOX_BF16, q=FAKE: L.vox_window_attn(
        q, ldq, FAKE, FAKE, 1280, 750, FAKE, FAKE, 3840, nq, FAKE, od, 1280, 32, hd, W, 0.158, None)
    assert w(q=None) == V.VOX_ERR_NULL
    assert w(W=0) == V.VOX_ERR_RANGE
    assert w(hd=65) == V.VOX_ERR_SHAPE
    assert w(ldq=1000) == V.VOX_ERR_SHAPE
    assert w(od=V.VOX_F16) == V.VOX_ERR_DTYPE
    r = L.vox_rmsnorm
    assert r(None, 1, 64, 64, 1e-5, None, FAKE, V.VOX_F32, 64, None) == V.VOX_ERR_NULL
    assert r(FAKE, 1, 64, 63, 1e-5, None, FAKE, V.VOX_F32, 64, None) == V.VOX_ERR_SHAPE
    assert r(FAKE, 1, 64, 64, -1.0, None, FAKE, V.VOX_F32, 64, None) == V.VOX_ERR_RANGE


def test_composed_validation(V):
    L = V.lib
    d = V.vox_decoder()
    assert L.vox_decoder_step(None, None) == V.VOX_ERR_NULL
    assert L.vox_decoder_step(ctypes.byref(d), None) == V.VOX_ERR_NULL
    e = V.vox_encoder()
    assert L.vox_encoder_chunk(ctypes.byref(e), None) == V.VOX_ERR_NULL


def test_product_path_fails_loudly_without_library(tmp_path, monkeypatch):
    """The binding refuses to import when libvox.so is absent (no fallback)."""
    import importlib.util
    import shutil

    pkg = tmp_path / "pkgcopy"
    pkg.mkdir()
    shutil.copy(os.path.join(ROOT, "bit_quantized_transformer_b200", "vox.py"), pkg / "vox.py")
    spec = importlib.util.spec_from_file_location("vox_copy", pkg / "vox.py")
    mod = importlib.util.module_from_spec(spec)
    with pytest.raises(ImportError):
        spec.loader.exec_module(mod)


def test_paged_attention_validation(V):
    """The batched paged attention rejects bad arguments on the host."""
    L = V.lib
    ws = V.vox_gqa_decode_attn_paged_workspace(4, 32, 8, 128, 8192)
    assert ws >= 4 * V.vox_gqa_decode_attn_workspace(32, 8, 128, 8192) - 256
    a = lambda nseq=4, nq=32, nkv=8, hd=128, W=8192, npg=600, pt=FAKE, wsp=FAKE, wsb=ws, kp=FAKE, out=FAKE: \
        L.vox_gqa_decode_attn_paged(FAKE, kp, FAKE, npg, pt, FAKE, nseq, out, nq, nkv, hd, W, 0.088, wsp, wsb, None)
    assert a(pt=None) == V.VOX_ERR_NULL
    assert a(kp=None) == V.VOX_ERR_NULL
    assert a(nseq=0) == V.VOX_ERR_RANGE
    assert a(nseq=65) == V.VOX_ERR_RANGE
    assert a(nq=30) == V.VOX_ERR_RANGE
    assert a(W=100) == V.VOX_ERR_RANGE               # not a multiple of the 64-slot page
    assert a(npg=0) == V.VOX_ERR_RANGE
    assert a(hd=64) == V.VOX_ERR_SHAPE
    assert a(npg=1 << 30) == V.VOX_ERR_SHAPE          # pool rows beyond 2^31
    assert a(wsp=None) == V.VOX_ERR_WORKSPACE
    assert a(wsb=ws - 16) == V.VOX_ERR_WORKSPACE
    assert a(kp=FAKE + 2) == V.VOX_ERR_ALIGN
    assert a(out=FAKE + 4) == V.VOX_ERR_ALIGN


def test_paged_append_epilogue_validation(V):
    L = V.lib
    w = V.vox_q4_weight(FAKE, 64, 96)
    ws = V.vox_q4_gemv_workspace(w, 2, None)

    def g(**kw):
        base = dict(op=V.VOX_EP_KV_APPEND_PAGED, k_cache=FAKE, v_cache=FAKE, n_kv_heads=1, head_dim=16,
                    window=64, q_rows=0, pos_dev=FAKE, page_table=FAKE, n_pages=4)
        base.update(kw)
        ep = V.vox_epilogue(**base)
        return L.vox_q4_gemv(ctypes.byref(w), FAKE, 2, 96, FAKE, 64, ctypes.byref(ep), FAKE, ws, None)

    assert g(page_table=None) == V.VOX_ERR_NULL
    assert g(pos_dev=None) == V.VOX_ERR_NULL
    assert g(window=96) == V.VOX_ERR_RANGE
    assert g(n_pages=0) == V.VOX_ERR_RANGE
    assert g(head_dim=32, q_rows=8) == V.VOX_ERR_SHAPE      # 8 + 2 * 32 rows > 64
    gm = lambda: L.vox_q4_gemm(ctypes.byref(V.vox_q4_weight(FAKE, 128, 128)), FAKE, V.VOX_BF16, 16, 128, FAKE,
                               V.VOX_F32, 128, ctypes.byref(V.vox_epilogue(op=V.VOX_EP_KV_APPEND_PAGED)), None)
    assert gm() == V.VOX_ERR_RANGE


def _fake_decoder(V, L=2, D=256, nq=4, nkv=2, hd=128, F=512, vocab=1024, W=128):
    """A decoder descriptor whose every pointer is FAKE (never dereferenced:
    the host checks below fail first) and whose weights have the right shapes."""
    keep = []
    Arr = V.vox_q4_weight * L
    QD, KVD = nq * hd, nkv * hd
    arrs = [Arr(*[V.vox_q4_weight(FAKE, n, k) for _ in range(L)])
            for n, k in ((QD + 2 * KVD, D), (D, QD), (2 * F, D), (D, F))]
    Ptr = ctypes.c_void_p * L
    caches = [Ptr(*[FAKE] * L), Ptr(*[FAKE] * L)]
    keep += arrs + caches
    d = V.vox_decoder()
    d.n_layers, d.dim, d.n_q_heads, d.n_kv_heads, d.head_dim, d.ffn, d.vocab, d.window = L, D, nq, nkv, hd, F, vocab, W
    d.eps = 1e-5
    d.wqkv, d.wo, d.w13, d.w2 = [ctypes.cast(a, ctypes.POINTER(V.vox_q4_weight)) for a in arrs]
    d.embedding = V.vox_q4_weight(FAKE, vocab, D)
    d.lm_head = V.vox_q4_weight(FAKE, vocab, D)
    d.k_cache, d.v_cache = [ctypes.cast(c, ctypes.POINTER(ctypes.c_void_p)) for c in caches]
    for name in ("token", "pos", "x", "h", "qkv", "attn", "act", "logits", "workspace"):
        setattr(d, name, FAKE)
    d.ws_bytes = 1 << 40
    return d, keep


def test_batch_fused_and_rope_validation(V):
    """Host checks of the batched step, the fused step and the RoPE setting:
    each bad field is refused before anything reaches the device."""
    L = V.lib
    d, keep = _fake_decoder(V)
    d.rope_theta = -1.0
    assert L.vox_decoder_step_kernels(ctypes.byref(d), None) == V.VOX_ERR_RANGE
    assert L.vox_decoder_step_fused(ctypes.byref(d), None) == V.VOX_ERR_RANGE
    d.rope_theta = float("nan")
    assert L.vox_decoder_step_fused(ctypes.byref(d), None) == V.VOX_ERR_RANGE
    d.rope_theta = 0.0
    d.attn = None
    assert L.vox_decoder_step_fused(ctypes.byref(d), None) == V.VOX_ERR_NULL
    d.attn = FAKE
    b = V.vox_decoder_batch()
    b.d = d
    b.n_seq, b.n_pages, b.page_table = 0, 10, FAKE
    assert L.vox_decoder_batch_step(ctypes.byref(b), None) == V.VOX_ERR_RANGE
    b.n_seq = 9
    assert L.vox_decoder_batch_step(ctypes.byref(b), None) == V.VOX_ERR_RANGE
    b.n_seq = 4
    b.page_table = None
    assert L.vox_decoder_batch_step(ctypes.byref(b), None) == V.VOX_ERR_NULL
    b.page_table = FAKE
    b.n_pages = 0
    assert L.vox_decoder_batch_step(ctypes.byref(b), None) == V.VOX_ERR_RANGE
    b.n_pages = 10
    b.d.window = 100                                  # not a multiple of the 64-slot page
    assert L.vox_decoder_batch_step(ctypes.byref(b), None) == V.VOX_ERR_RANGE
    b.d.window = 128
    b.d.rope_theta = -2.0
    assert L.vox_decoder_batch_step(ctypes.byref(b), None) == V.VOX_ERR_RANGE
    assert L.vox_decoder_batch_workspace(None) == 0
    ep = V.vox_epilogue(op=V.VOX_EP_RESIDUAL, residual=FAKE, ldr=64, rope_theta=1e4)   # RoPE only with an append
    w = V.vox_q4_weight(FAKE, 64, 96)
    assert L.vox_q4_gemv(ctypes.byref(w), FAKE, 1, 96, FAKE, 64, ctypes.byref(ep), FAKE, 256, None) == V.VOX_ERR_RANGE
    ep = V.vox_epilogue(op=V.VOX_EP_KV_APPEND, k_cache=FAKE, v_cache=FAKE, n_kv_heads=1, head_dim=24, window=4,
                        q_rows=0, pos=0, rope_theta=1e4)                             # head_dim not a multiple of 16
    assert L.vox_q4_gemv(ctypes.byref(w), FAKE, 1, 96, FAKE, 64, ctypes.byref(ep), FAKE, 256, None) == V.VOX_ERR_RANGE


def test_encoder_streaming_validation(V):
    """A streamed chunk refuses a next history that is one of its inputs."""
    L = V.lib
    Ln = 1
    Arr = V.vox_q4_weight * Ln
    D, F, R = 1280, 5120, 256
    arrs = [Arr(V.vox_q4_weight(FAKE, n, k)) for n, k in ((3 * D, D), (D, D), (F, D), (D, F))]
    Ptr = ctypes.c_void_p * Ln
    kh, vh = Ptr(FAKE), Ptr(FAKE + 4096)
    e = V.vox_encoder()
    e.n_layers, e.dim, e.n_heads, e.head_dim, e.ffn, e.window, e.rows, e.adapter_out = Ln, D, 32, 40, F, 750, R, 3072
    e.eps = 1e-5
    e.wqkv, e.wo, e.wup, e.wdown = [ctypes.cast(a, ctypes.POINTER(V.vox_q4_weight)) for a in arrs]
    e.adapter = V.vox_q4_weight(FAKE, 3072, 4 * D)
    e.adapter2 = V.vox_q4_weight(FAKE, 3072, 3072)
    e.k_hist, e.v_hist = ctypes.cast(kh, ctypes.POINTER(ctypes.c_void_p)), ctypes.cast(vh, ctypes.POINTER(ctypes.c_void_p))
    for name in ("x", "xn", "qkv", "att", "up", "adapter_mid", "adapter_out_buf"):
        setattr(e, name, FAKE)
    kn_alias, vn = Ptr(FAKE), Ptr(FAKE + 8192)
    e.k_hist_next = ctypes.cast(kn_alias, ctypes.POINTER(ctypes.c_void_p))
    e.v_hist_next = ctypes.cast(vn, ctypes.POINTER(ctypes.c_void_p))
    assert L.vox_encoder_chunk(ctypes.byref(e), None) == V.VOX_ERR_ALIGN
    e.v_hist_next = None
    assert L.vox_encoder_chunk(ctypes.byref(e), None) == V.VOX_ERR_NULL
