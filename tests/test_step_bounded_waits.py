"""The persistent decoder step's bounded device-side waits, made to run out
without faulting or hanging the GPU.

With the test hook VOX_TEST_WITHHOLD_STAGE=1 (read by vox_decoder_step at
launch), warp 0 of CTA 0 first waits on an mbarrier that nothing ever
completes.  That wait gives up after about one second, records 0x530 in the
device status word and raises the abort flag, so every other CTA leaves its
grid barrier early; the launch returns and the context stays usable.  After the workspace
is zeroed again and the state restored, the next step is correct."""
import os
import time

import numpy as np
import pytest

import synth
from oracle import ref

pytestmark = pytest.mark.gpu
TOL = 2e-3
HOOK = "VOX_TEST_WITHHOLD_STAGE"


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


def test_withheld_stage_gives_up_and_the_step_returns(env):
    torch, V, WL = env
    shape = synth.DecoderShape(n_layers=2, dim=256, n_q_heads=4, n_kv_heads=2, head_dim=128, ffn=512, vocab=1024,
                               window=64)
    dm = WL.DecoderModel(shape, seed=5, filled=70, token=3)
    torch.cuda.synchronize()
    assert V.vox_device_status(True) == 0
    os.environ[HOOK] = "1"
    try:
        t0 = time.monotonic()
        dm.step()
        torch.cuda.synchronize()
        dt = time.monotonic() - t0
    finally:
        del os.environ[HOOK]
    assert V.vox_device_status(True) == 0x530
    assert dt < 30.0, dt                               # one bounded wait, then every CTA leaves

    # the context is still usable: restore the state and step again
    dm.workspace.zero_()
    for l in range(dm.L):
        kb, vb = synth.decoder_layer_cache(shape, l, 5, dm.W)
        dm.k_cache[l].copy_(WL.bf16_dev(kb, "cuda"))
        dm.v_cache[l].copy_(WL.bf16_dev(vb, "cuda"))
    dm.pos.fill_(70)
    dm.token.fill_(3)
    dm.step()
    torch.cuda.synchronize()
    assert V.vox_device_status(True) == 0
    assert int(dm.pos.item()) == 71
    logits = dm.logits.cpu().numpy()
    lq, ld = synth.q4_blocks(shape.vocab, shape.dim, 5, synth.LM_HEAD_ID)
    xf = ref.rmsnorm(dm.x.cpu().numpy())
    W = ref.q4_weights(lq, ld)
    assert ref.gemv_error(logits[None], xf[None] @ W.T, xf[None], W) <= TOL
    assert int(dm.token.item()) == int(np.argmax(logits))
