"""vox_gqa_decode_attn_static, the entry point that allocates nothing.

It serves callers that cannot hand the library device scratch (a host
program that links only this C library and owns no device allocator; a
real-time audio thread that must not call cudaMalloc, which can block and
synchronise the device).  Its split-KV records live in one fixed array inside
the loaded library.  These tests call it through the C ABI and check:

* on the decoder's shape (32 query / 8 kv heads x 128, 8192-slot rolling
  cache), two calls in a row at different positions (the second after the
  window has wrapped): the output equals the workspace entry point's bit for
  bit (same kernels, same grid, deterministic combine) and is within the
  attention tolerance of the fp64 oracle;
* every documented shape (1..8 kv heads, groups of 1, 2 and 4) on seeded
  random caches, against the workspace entry point (bit for bit) and the
  oracle, including 7 kv heads x 4 at the full 8192-slot window, the shape
  that needs the most records;
* shapes beyond the array are refused with VOX_ERR_RANGE.

The file sorts last so that it also runs after every other GPU test."""
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


def run_both(env, q, kb, vb, n_q, n_kv, W, pos):
    """Static and workspace entry points on the same inputs; the workspace
    starts filled with 0xFF bytes (its contract needs no initial contents)."""
    torch, V, WL = env
    hd = 128
    kc, vc = WL.bf16_dev(kb, "cuda"), WL.bf16_dev(vb, "cuda")
    qd = WL.to_dev(q, "cuda")
    wsb = V.vox_gqa_decode_attn_workspace(n_q, n_kv, hd, W)
    ws = torch.full((wsb,), 0xFF, dtype=torch.uint8, device="cuda")
    out_ws = torch.full((n_q, hd), float("nan"), device="cuda")
    out_st = torch.full((n_q, hd), float("nan"), device="cuda")
    scale = 1.0 / math.sqrt(hd)
    V.vox_gqa_decode_attn(qd, kc, vc, out_ws, n_q, n_kv, hd, W, pos, scale, ws, wsb)
    V.vox_gqa_decode_attn_static(qd, kc, vc, out_st, n_q, n_kv, hd, W, pos, scale)
    torch.cuda.synchronize()
    assert V.vox_device_status(True) == 0
    return out_st.cpu().numpy(), out_ws.cpu().numpy()


def oracle_err(o, q, kb, vb, n_q, n_kv, W, pos):
    nv = min(pos + 1, W)
    o_ref = ref.c_gqa_attn(q, kb, vb, pos)
    return ref.attn_error(o, o_ref, ref.attn_probs(q, kb, pos), ref.bf16_to_f64(vb[:, :nv]), n_q // n_kv)


def test_static_scratch_matches_workspace_entry(env):
    n_q, n_kv, hd, W = 32, 8, 128, 8192
    kb = synth.bf16_normal((n_kv, W, hd), 0, 61)
    vb = synth.bf16_normal((n_kv, W, hd), 0, 62)
    for call, pos in enumerate((1500, W + 300)):
        q = synth.activations(n_q, hd, 0, 63 + call) * 2.0
        o_st, o_ws = run_both(env, q, kb, vb, n_q, n_kv, W, pos)
        assert np.all(np.isfinite(o_st))
        assert np.array_equal(o_st.view(np.uint32), o_ws.view(np.uint32)), call
        err = oracle_err(o_st, q, kb, vb, n_q, n_kv, W, pos)
        assert err <= TOL, (call, err)


def test_static_scratch_takes_every_documented_shape(env):
    """Every kv head count up to 8 with groups up to 4 fits the array and
    gives the workspace entry point's output bit for bit, within the oracle's
    tolerance; 7 kv heads x 4 also at the full window."""
    cases = [(n_kv, group, 1024, 1500) for n_kv in range(1, 9) for group in (1, 2, 4)]
    cases.append((7, 4, 8192, 8192 + 300))
    for n_kv, group, W, pos in cases:
        n_q = n_kv * group
        tid = 700 + 4 * (n_kv * 8 + group) + (W > 1024)
        kb = synth.bf16_normal((n_kv, W, 128), 0, tid)
        vb = synth.bf16_normal((n_kv, W, 128), 0, tid + 1)
        q = synth.activations(n_q, 128, 0, tid + 2)
        o_st, o_ws = run_both(env, q, kb, vb, n_q, n_kv, W, pos)
        assert np.array_equal(o_st.view(np.uint32), o_ws.view(np.uint32)), (n_kv, group, W)
        err = oracle_err(o_st, q, kb, vb, n_q, n_kv, W, pos)
        assert err <= TOL, (n_kv, group, W, err)


def test_static_scratch_rejects_shapes_beyond_its_size(env):
    torch, V, WL = env
    q = torch.zeros(64, 128, device="cuda")
    c = torch.zeros(16, 64, 128, dtype=torch.bfloat16, device="cuda")
    out = torch.empty(64, 128, device="cuda")
    for n_q, n_kv in ((64, 16), (64, 8)):            # 16 kv heads; groups of 8
        st = V.lib.vox_gqa_decode_attn_static(q.data_ptr(), c.data_ptr(), c.data_ptr(), out.data_ptr(), n_q, n_kv,
                                              128, 64, 10, 0.1, None)
        assert st == V.VOX_ERR_RANGE
        assert b"static scratch" in V.lib.vox_last_error()
