"""vox_gqa_decode_attn_static, the entry point that allocates nothing, against
vox_gqa_decode_attn with a caller workspace: the same decoder-shaped inputs
(32 query / 8 kv heads x 128, 8192-slot rolling cache), two calls in a row at
different positions (the second after the window has wrapped), each within
the attention tolerance of the workspace entry point's output.  The file
sorts last so that it also runs after every other GPU test."""
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


def test_static_scratch_matches_workspace_entry(env):
    torch, V, WL = env
    n_q, n_kv, hd, W = 32, 8, 128, 8192
    kb = synth.bf16_normal((n_kv, W, hd), 0, 61)
    vb = synth.bf16_normal((n_kv, W, hd), 0, 62)
    kc, vc = WL.bf16_dev(kb, "cuda"), WL.bf16_dev(vb, "cuda")
    wsb = V.vox_gqa_decode_attn_workspace(n_q, n_kv, hd, W)
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    scale = 1.0 / math.sqrt(hd)
    for call, pos in enumerate((1500, W + 300)):
        q = synth.activations(n_q, hd, 0, 63 + call) * 2.0
        qd = WL.to_dev(q, "cuda")
        out_ws = torch.empty(n_q, hd, device="cuda")
        out_st = torch.full((n_q, hd), float("nan"), device="cuda")
        V.vox_gqa_decode_attn(qd, kc, vc, out_ws, n_q, n_kv, hd, W, pos, scale, ws, wsb)
        V.vox_gqa_decode_attn_static(qd, kc, vc, out_st, n_q, n_kv, hd, W, pos, scale)
        torch.cuda.synchronize()
        assert V.vox_device_status(True) == 0
        o_ws = out_ws.cpu().numpy()
        o_st = out_st.cpu().numpy()
        assert np.all(np.isfinite(o_st))
        nv = min(pos + 1, W)
        err = ref.attn_error(o_st, o_ws.astype(np.float64), ref.attn_probs(q, kb, pos),
                             ref.bf16_to_f64(vb[:, :nv]), n_q // n_kv)
        assert err <= TOL, (call, err)


def test_static_scratch_takes_every_documented_shape(env):
    """Every kv head count up to 8 with groups up to 4 fits the array (a
    small window, so each call is quick); 16 kv heads or groups of 8 do not."""
    torch, V, WL = env
    W, hd = 64, 128
    c = torch.zeros(8, W, hd, dtype=torch.bfloat16, device="cuda")
    for n_kv in range(1, 9):
        for group in (1, 2, 4):
            q = torch.zeros(n_kv * group, hd, device="cuda")
            out = torch.empty(n_kv * group, hd, device="cuda")
            V.vox_gqa_decode_attn_static(q, c, c, out, n_kv * group, n_kv, hd, W, 10, 0.1)
    torch.cuda.synchronize()
    assert V.vox_device_status(True) == 0
    q = torch.zeros(64, hd, device="cuda")
    out = torch.empty(64, hd, device="cuda")
    st = V.lib.vox_gqa_decode_attn_static(q.data_ptr(), c.data_ptr(), c.data_ptr(), out.data_ptr(), 64, 8, hd, W,
                                          10, 0.1, None)
    assert st == V.VOX_ERR_RANGE


def test_static_scratch_rejects_shapes_beyond_its_size(env):
    torch, V, WL = env
    q = torch.zeros(64, 128, device="cuda")
    c = torch.zeros(16, 64, 128, dtype=torch.bfloat16, device="cuda")
    out = torch.empty(64, 128, device="cuda")
    st = V.lib.vox_gqa_decode_attn_static(q.data_ptr(), c.data_ptr(), c.data_ptr(), out.data_ptr(), 64, 16, 128,
                                          64, 10, 0.1, None)
    assert st == V.VOX_ERR_RANGE
    assert b"static scratch" in V.lib.vox_last_error()
