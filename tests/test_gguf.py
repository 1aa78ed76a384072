"""The GGUF reader (vox_gguf_*): metadata and tensors of synthetic files
written by tests/gguf_writer.py from the container's layout, the error codes
of malformed files, and (on the GPU) a Q4_0 tensor uploaded and repacked,
then dequantised bit for bit against the oracle."""
import numpy as np
import pytest

import synth
from oracle import ref
import gguf_writer as GW


@pytest.fixture(scope="module")
def V():
    from bit_quantized_transformer_b200 import build

    build.build()
    from bit_quantized_transformer_b200 import vox

    return vox


def sample_file(path, alignment=64):
    qs, d = synth.q4_blocks(40, 96, 0, 4242)
    q4 = synth.gguf_bytes(qs, d).tobytes()
    f32 = np.arange(10, dtype=np.float32) * 0.5
    f16 = (np.arange(6, dtype=np.float32) - 2.5).astype(np.float16)
    meta = [("general.architecture", GW.STR, "voxtral"), ("dec.block_count", GW.U32, 26),
            ("dec.neg", GW.I32, -7), ("dec.big", GW.U64, 2 ** 40), ("dec.eps", GW.F32, 1e-5),
            ("dec.theta", GW.F64, 1.0e6), ("dec.flag", GW.BOOL, 1), ("dec.i8", GW.I8, -3),
            ("dec.u16", GW.U16, 65535), ("tok.list", GW.ARR, (GW.STR, ["a", "bc", ""])),
            ("tok.ids", GW.ARR, (GW.I32, [1, 2, 3, 4]))]
    tensors = [("blk.0.wq", [96, 40], 2, q4), ("norm", [10], 0, f32.tobytes()), ("emb.f16", [3, 2], 1, f16.tobytes()),
               ("other.q8", [32, 2], 8, b"\x01" * 68)]
    GW.write_gguf(path, meta, tensors, alignment=alignment)
    return qs, d, q4, f32, f16


def test_gguf_metadata_and_tensors(V, tmp_path):
    path = tmp_path / "m.gguf"
    qs, d, q4, f32, f16 = sample_file(path)
    g = V.GGUF(path)
    assert g.tensor_count() == 4
    assert g.info(0) == ("blk.0.wq", 2, [96, 40], 40 * 3 * 18)
    assert g.info(1) == ("norm", 0, [10], 40)
    assert g.info(2) == ("emb.f16", 1, [3, 2], 12)
    assert g.info(3)[3] == 0                                  # a type this library does not read
    assert g.data(0) == q4
    assert np.array_equal(np.frombuffer(g.data(1), np.float32), f32)
    assert np.array_equal(np.frombuffer(g.data(2), np.float16), f16)
    assert g.find("norm") == 1 and g.find("missing") == -1
    assert g.get_string("general.architecture") == "voxtral"
    assert g.get_int("dec.block_count") == 26
    assert g.get_int("dec.neg") == -7
    assert g.get_int("dec.big") == 2 ** 40
    assert g.get_int("dec.flag") == 1 and g.get_int("dec.i8") == -3 and g.get_int("dec.u16") == 65535
    assert abs(g.get_float("dec.eps") - 1e-5) < 1e-12
    assert g.get_float("dec.theta") == 1.0e6
    with pytest.raises(V.VoxError):
        g.get_int("missing.key")
    with pytest.raises(V.VoxError):
        g.get_int("dec.eps")                                   # a float, not an int
    assert g.get_string("dec.block_count") is None
    g.close()


@pytest.mark.parametrize("case", ["magic", "version", "misaligned", "past_end", "truncated_header"])
def test_gguf_malformed_files(V, tmp_path, case):
    path = tmp_path / f"{case}.gguf"
    qs, d = synth.q4_blocks(16, 64, 0, 1)
    q4 = synth.gguf_bytes(qs, d).tobytes()
    tensors = [("w", [64, 16], 2, q4)]
    want = {"magic": V.VOX_ERR_SHAPE, "version": V.VOX_ERR_SHAPE, "misaligned": V.VOX_ERR_ALIGN,
            "past_end": V.VOX_ERR_RANGE, "truncated_header": V.VOX_ERR_SHAPE}[case]
    if case == "magic":
        GW.write_gguf(path, [], tensors, magic=b"GGUG")
    elif case == "version":
        GW.write_gguf(path, [], tensors, version=7)
    elif case == "misaligned":
        GW.write_gguf(path, [], tensors, bad_offset=(0, 8))
    elif case == "past_end":
        start = GW.write_gguf(path, [], tensors)
        GW.write_gguf(path, [], tensors, truncate=start + len(q4) - 1)
    else:
        GW.write_gguf(path, [("k", GW.STR, "value")], tensors, truncate=30)
    import ctypes

    h = ctypes.c_void_p()
    assert V.lib.vox_gguf_open(str(path).encode(), ctypes.byref(h)) == want
    assert not h.value


@pytest.mark.gpu
def test_gguf_upload_q4_dequant_bitexact(V, tmp_path):
    import torch

    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    path = tmp_path / "m.gguf"
    qs, d, q4, _, _ = sample_file(path)
    g = V.GGUF(path)
    i = g.find("blk.0.wq")
    scratch = torch.empty(len(q4), dtype=torch.uint8, device="cuda")
    packed = torch.empty(V.vox_q4_packed_bytes(40, 96), dtype=torch.uint8, device="cuda")
    g.upload_q4(i, scratch, packed)
    w = V.weight(packed, 40, 96)
    out = torch.empty(40, 96, dtype=torch.float32, device="cuda")
    V.vox_q4_dequant(w, 0, 40, out, V.VOX_F32, 96)
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy(), ref.c_dequant_f32(qs, d))
    with pytest.raises(V.VoxError):
        g.upload_q4(g.find("norm"), scratch, packed)          # not Q4_0
    g.close()
