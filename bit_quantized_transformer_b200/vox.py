"""Thin Python binding of libvox (include/vox.h).

Argument marshalling only: every function here has the name of the C entry
point it calls, converts torch tensors to raw device addresses and raises
:class:`VoxError` on a non-OK status.  All computation runs in libvox's
kernels; there is no fallback.  Importing this module loads libvox.so and
fails loudly if it is missing (build it with ``python -m
bit_quantized_transformer_b200.build``).
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libvox.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libvox.so not found at {LIB_PATH}; build it with "
                      "`python -m bit_quantized_transformer_b200.build`")
lib = ctypes.CDLL(LIB_PATH)

# status codes and enums (include/vox.h)
VOX_OK, VOX_ERR_NULL, VOX_ERR_SHAPE, VOX_ERR_ALIGN, VOX_ERR_DTYPE = 0, 1, 2, 3, 4
VOX_ERR_RANGE, VOX_ERR_WORKSPACE, VOX_ERR_TIMEOUT, VOX_ERR_CUDA = 5, 6, 7, 8
VOX_F32, VOX_BF16, VOX_F16 = 0, 1, 2
VOX_PACK_PLAIN, VOX_PACK_GATE_UP = 0, 1
VOX_EP_NONE, VOX_EP_RESIDUAL, VOX_EP_SILU_MUL, VOX_EP_GELU, VOX_EP_KV_APPEND, VOX_EP_ARGMAX, VOX_EP_KV_APPEND_PAGED = range(7)

_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_I64 = ctypes.c_int64
_F = ctypes.c_float
_SZ = ctypes.c_size_t


class vox_q4_weight(ctypes.Structure):
    _fields_ = [("data", _P), ("n", _I64), ("k", _I64)]


class vox_epilogue(ctypes.Structure):
    _fields_ = [("op", _I32), ("rmsnorm", _I32), ("eps", _F), ("norm_weight", _P),
                ("residual", _P), ("ldr", _I64), ("k_cache", _P), ("v_cache", _P),
                ("n_kv_heads", _I32), ("head_dim", _I32), ("window", _I32), ("q_rows", _I32),
                ("pos", _I64), ("pos_dev", _P), ("argmax", _P), ("page_table", _P), ("n_pages", _I64),
                ("rope_theta", _F)]


class vox_decoder(ctypes.Structure):
    _fields_ = [("n_layers", _I32), ("dim", _I32), ("n_q_heads", _I32), ("n_kv_heads", _I32),
                ("head_dim", _I32), ("ffn", _I32), ("vocab", _I32), ("window", _I32), ("eps", _F),
                ("wqkv", ctypes.POINTER(vox_q4_weight)), ("wo", ctypes.POINTER(vox_q4_weight)),
                ("w13", ctypes.POINTER(vox_q4_weight)), ("w2", ctypes.POINTER(vox_q4_weight)),
                ("embedding", vox_q4_weight), ("lm_head", vox_q4_weight),
                ("k_cache", ctypes.POINTER(_P)), ("v_cache", ctypes.POINTER(_P)),
                ("token", _P), ("pos", _P), ("x", _P), ("h", _P), ("qkv", _P), ("attn", _P),
                ("act", _P), ("logits", _P), ("workspace", _P), ("ws_bytes", _SZ), ("rope_theta", _F)]


class vox_decoder_batch(ctypes.Structure):
    _fields_ = [("d", vox_decoder), ("n_seq", _I32), ("n_pages", _I64), ("page_table", _P)]


class vox_encoder(ctypes.Structure):
    _fields_ = [("n_layers", _I32), ("dim", _I32), ("n_heads", _I32), ("head_dim", _I32),
                ("ffn", _I32), ("window", _I32), ("rows", _I32), ("adapter_out", _I32), ("eps", _F),
                ("wqkv", ctypes.POINTER(vox_q4_weight)), ("wo", ctypes.POINTER(vox_q4_weight)),
                ("wup", ctypes.POINTER(vox_q4_weight)), ("wdown", ctypes.POINTER(vox_q4_weight)),
                ("adapter", vox_q4_weight), ("adapter2", vox_q4_weight),
                ("k_hist", ctypes.POINTER(_P)), ("v_hist", ctypes.POINTER(_P)),
                ("x", _P), ("xn", _P), ("qkv", _P), ("att", _P), ("up", _P), ("adapter_mid", _P),
                ("adapter_out_buf", _P), ("tap", _P), ("k_hist_next", ctypes.POINTER(_P)),
                ("v_hist_next", ctypes.POINTER(_P))]


_W = ctypes.POINTER(vox_q4_weight)
_E = ctypes.POINTER(vox_epilogue)
_SIGS = {
    "vox_status_str": (ctypes.c_char_p, [_I32]),
    "vox_last_error": (ctypes.c_char_p, []),
    "vox_device_status": (_I32, [_I32]),
    "vox_q4_packed_bytes": (_I64, [_I64, _I64]),
    "vox_q4_pack": (_I32, [_P, _I64, _I64, _I32, _P, _P]),
    "vox_q4_dequant": (_I32, [_W, _I64, _I64, _P, _I32, _I64, _P]),
    "vox_q4_gemv": (_I32, [_W, _P, _I64, _I64, _P, _I64, _E, _P, _SZ, _P]),
    "vox_q4_gemv_workspace": (_SZ, [_W, _I64, _E]),
    "vox_q4_gemm": (_I32, [_W, _P, _I32, _I64, _I64, _P, _I32, _I64, _E, _P]),
    "vox_q4_matmul": (_I32, [_W, _P, _I64, _I64, _P, _I64, _E, _P, _SZ, _P]),
    "vox_q4_matmul_workspace": (_SZ, [_W, _I64, _E]),
    "vox_kv_append_rolling": (_I32, [_P, _P, _P, _P, _I32, _I32, _I32, _I32, _I64, _P]),
    "vox_gqa_decode_attn": (_I32, [_P, _P, _P, _P, _I32, _I32, _I32, _I32, _I64, _F, _P, _SZ, _P]),
    "vox_gqa_decode_attn_workspace": (_SZ, [_I32, _I32, _I32, _I32]),
    "vox_gqa_decode_attn_static": (_I32, [_P, _P, _P, _P, _I32, _I32, _I32, _I32, _I64, _F, _P]),
    "vox_gqa_decode_attn_paged": (_I32, [_P, _P, _P, _I64, _P, _P, _I32, _P, _I32, _I32, _I32, _I32, _F, _P, _SZ,
                                         _P]),
    "vox_gqa_decode_attn_paged_workspace": (_SZ, [_I32, _I32, _I32, _I32, _I32]),
    "vox_window_attn": (_I32, [_P, _I64, _P, _P, _I64, _I64, _P, _P, _I64, _I64, _P, _I32, _I64,
                               _I32, _I32, _I32, _F, _P]),
    "vox_rmsnorm": (_I32, [_P, _I64, _I64, _I64, _F, _P, _P, _I32, _I64, _P]),
    "vox_decoder_workspace": (_SZ, [ctypes.POINTER(vox_decoder)]),
    "vox_decoder_step": (_I32, [ctypes.POINTER(vox_decoder), _P]),
    "vox_decoder_step_kernels": (_I32, [ctypes.POINTER(vox_decoder), _P]),
    "vox_decoder_step_fused": (_I32, [ctypes.POINTER(vox_decoder), _P]),
    "vox_decoder_batch_workspace": (_SZ, [ctypes.POINTER(vox_decoder_batch)]),
    "vox_decoder_batch_step": (_I32, [ctypes.POINTER(vox_decoder_batch), _P]),
    "vox_encoder_chunk": (_I32, [ctypes.POINTER(vox_encoder), _P]),
    "vox_gguf_open": (_I32, [ctypes.c_char_p, ctypes.POINTER(_P)]),
    "vox_gguf_close": (None, [_P]),
    "vox_gguf_tensor_count": (_I64, [_P]),
    "vox_gguf_find_tensor": (_I64, [_P, ctypes.c_char_p]),
    "vox_gguf_tensor_info": (_I32, [_P, _I64, ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(_I32),
                                    ctypes.POINTER(_I32), ctypes.POINTER(_I64), ctypes.POINTER(ctypes.c_uint64)]),
    "vox_gguf_tensor_data": (_P, [_P, _I64]),
    "vox_gguf_get_int": (_I32, [_P, ctypes.c_char_p, ctypes.POINTER(_I64)]),
    "vox_gguf_get_float": (_I32, [_P, ctypes.c_char_p, ctypes.POINTER(ctypes.c_double)]),
    "vox_gguf_get_string": (ctypes.c_char_p, [_P, ctypes.c_char_p]),
    "vox_gguf_upload_q4": (_I32, [_P, _I64, _P, _SZ, _I32, _P, _P]),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


class VoxError(RuntimeError):
    def __init__(self, status: int, where: str):
        name = lib.vox_status_str(status).decode()
        detail = lib.vox_last_error().decode() if status == VOX_ERR_CUDA else ""
        super().__init__(f"{where}: {name}" + (f" ({detail})" if detail else ""))
        self.status = status


def _check(st: int, where: str) -> None:
    if st != VOX_OK:
        raise VoxError(st, where)


def ptr(t) -> int | None:
    """Raw address of a tensor (or an int address, or None)."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def stream_ptr(stream=None) -> int | None:
    """cudaStream_t of a torch stream (default: torch's current stream)."""
    import torch

    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def weight(packed, n: int, k: int) -> vox_q4_weight:
    return vox_q4_weight(ptr(packed), n, k)


# ------------------------------------------------------------ entry points
def vox_q4_packed_bytes(n: int, k: int) -> int:
    return lib.vox_q4_packed_bytes(n, k)


def vox_q4_pack(gguf, n, k, flags, packed, stream=None):
    _check(lib.vox_q4_pack(ptr(gguf), n, k, flags, ptr(packed), stream_ptr(stream)), "vox_q4_pack")


def vox_q4_dequant(w: vox_q4_weight, row0, nrows, out, out_dtype, ldo, stream=None):
    _check(lib.vox_q4_dequant(ctypes.byref(w), row0, nrows, ptr(out), out_dtype, ldo, stream_ptr(stream)),
           "vox_q4_dequant")


def vox_q4_gemv_workspace(w: vox_q4_weight, m: int, ep: vox_epilogue | None = None) -> int:
    return lib.vox_q4_gemv_workspace(ctypes.byref(w), m, ctypes.byref(ep) if ep is not None else None)


def vox_q4_gemv(w: vox_q4_weight, x, m, ldx, y, ldy, ep=None, workspace=None, ws_bytes=0, stream=None):
    _check(lib.vox_q4_gemv(ctypes.byref(w), ptr(x), m, ldx, ptr(y), ldy,
                           ctypes.byref(ep) if ep is not None else None, ptr(workspace), ws_bytes,
                           stream_ptr(stream)), "vox_q4_gemv")


def vox_q4_gemm(w: vox_q4_weight, x, x_dtype, m, ldx, y, y_dtype, ldy, ep=None, stream=None):
    _check(lib.vox_q4_gemm(ctypes.byref(w), ptr(x), x_dtype, m, ldx, ptr(y), y_dtype, ldy,
                           ctypes.byref(ep) if ep is not None else None, stream_ptr(stream)), "vox_q4_gemm")


def vox_q4_matmul_workspace(w: vox_q4_weight, m: int, ep: vox_epilogue | None = None) -> int:
    return lib.vox_q4_matmul_workspace(ctypes.byref(w), m, ctypes.byref(ep) if ep is not None else None)


def vox_q4_matmul(w: vox_q4_weight, x, m, ldx, y, ldy, ep=None, workspace=None, ws_bytes=0, stream=None):
    _check(lib.vox_q4_matmul(ctypes.byref(w), ptr(x), m, ldx, ptr(y), ldy,
                             ctypes.byref(ep) if ep is not None else None, ptr(workspace), ws_bytes,
                             stream_ptr(stream)), "vox_q4_matmul")


def vox_kv_append_rolling(k_cache, v_cache, k_new, v_new, new_dtype, n_kv_heads, head_dim, window, pos,
                          stream=None):
    _check(lib.vox_kv_append_rolling(ptr(k_cache), ptr(v_cache), ptr(k_new), ptr(v_new), new_dtype,
                                     n_kv_heads, head_dim, window, pos, stream_ptr(stream)),
           "vox_kv_append_rolling")


def vox_gqa_decode_attn_workspace(n_q_heads, n_kv_heads, head_dim, window) -> int:
    return lib.vox_gqa_decode_attn_workspace(n_q_heads, n_kv_heads, head_dim, window)


def vox_gqa_decode_attn(q, k_cache, v_cache, out, n_q_heads, n_kv_heads, head_dim, window, pos, scale,
                        workspace, ws_bytes, stream=None):
    _check(lib.vox_gqa_decode_attn(ptr(q), ptr(k_cache), ptr(v_cache), ptr(out), n_q_heads, n_kv_heads,
                                   head_dim, window, pos, scale, ptr(workspace), ws_bytes, stream_ptr(stream)),
           "vox_gqa_decode_attn")


def vox_gqa_decode_attn_paged_workspace(n_seq, n_q_heads, n_kv_heads, head_dim, window) -> int:
    return lib.vox_gqa_decode_attn_paged_workspace(n_seq, n_q_heads, n_kv_heads, head_dim, window)


def vox_gqa_decode_attn_paged(q, k_pool, v_pool, n_pages, page_table, pos, n_seq, out, n_q_heads, n_kv_heads,
                              head_dim, window, scale, workspace, ws_bytes, stream=None):
    _check(lib.vox_gqa_decode_attn_paged(ptr(q), ptr(k_pool), ptr(v_pool), n_pages, ptr(page_table), ptr(pos), n_seq,
                                         ptr(out), n_q_heads, n_kv_heads, head_dim, window, scale, ptr(workspace),
                                         ws_bytes, stream_ptr(stream)),
           "vox_gqa_decode_attn_paged")


def vox_gqa_decode_attn_static(q, k_cache, v_cache, out, n_q_heads, n_kv_heads, head_dim, window, pos, scale,
                               stream=None):
    _check(lib.vox_gqa_decode_attn_static(ptr(q), ptr(k_cache), ptr(v_cache), ptr(out), n_q_heads, n_kv_heads,
                                          head_dim, window, pos, scale, stream_ptr(stream)),
           "vox_gqa_decode_attn_static")


def vox_window_attn(q, ldq, k_hist, v_hist, ld_hist, n_hist, k_new, v_new, ld_new, n_q, out, out_dtype, ldo,
                    n_heads, head_dim, window, scale, stream=None):
    _check(lib.vox_window_attn(ptr(q), ldq, ptr(k_hist), ptr(v_hist), ld_hist, n_hist, ptr(k_new), ptr(v_new),
                               ld_new, n_q, ptr(out), out_dtype, ldo, n_heads, head_dim, window, scale,
                               stream_ptr(stream)), "vox_window_attn")


def vox_rmsnorm(x, m, n, ldx, eps, g, out, out_dtype, ldo, stream=None):
    _check(lib.vox_rmsnorm(ptr(x), m, n, ldx, eps, ptr(g), ptr(out), out_dtype, ldo, stream_ptr(stream)),
           "vox_rmsnorm")


def vox_decoder_workspace(dec: vox_decoder) -> int:
    return lib.vox_decoder_workspace(ctypes.byref(dec))


def vox_decoder_step(dec: vox_decoder, stream=None):
    _check(lib.vox_decoder_step(ctypes.byref(dec), stream_ptr(stream)), "vox_decoder_step")


def vox_decoder_step_kernels(dec: vox_decoder, stream=None):
    _check(lib.vox_decoder_step_kernels(ctypes.byref(dec), stream_ptr(stream)), "vox_decoder_step_kernels")


def vox_decoder_step_fused(dec: vox_decoder, stream=None):
    _check(lib.vox_decoder_step_fused(ctypes.byref(dec), stream_ptr(stream)), "vox_decoder_step_fused")


def vox_decoder_batch_workspace(b: vox_decoder_batch) -> int:
    return lib.vox_decoder_batch_workspace(ctypes.byref(b))


def vox_decoder_batch_step(b: vox_decoder_batch, stream=None):
    _check(lib.vox_decoder_batch_step(ctypes.byref(b), stream_ptr(stream)), "vox_decoder_batch_step")


def vox_encoder_chunk(enc: vox_encoder, stream=None):
    _check(lib.vox_encoder_chunk(ctypes.byref(enc), stream_ptr(stream)), "vox_encoder_chunk")


def vox_device_status(clear: bool = True) -> int:
    return lib.vox_device_status(1 if clear else 0)


# ------------------------------------------------------------ GGUF files
class GGUF:
    """A GGUF file opened through vox_gguf_open (the handle is closed with
    close() or when the object is collected)."""

    def __init__(self, path: str):
        h = _P()
        _check(lib.vox_gguf_open(str(path).encode(), ctypes.byref(h)), "vox_gguf_open")
        self.h = h

    def close(self):
        if self.h:
            lib.vox_gguf_close(self.h)
            self.h = None

    def __del__(self):
        self.close()

    def tensor_count(self) -> int:
        return lib.vox_gguf_tensor_count(self.h)

    def find(self, name: str) -> int:
        return lib.vox_gguf_find_tensor(self.h, name.encode())

    def info(self, i: int):
        """(name, type, dims innermost first, nbytes) of tensor i."""
        name, typ, nd = ctypes.c_char_p(), _I32(), _I32()
        dims, nb = (_I64 * 4)(), ctypes.c_uint64()
        _check(lib.vox_gguf_tensor_info(self.h, i, ctypes.byref(name), ctypes.byref(typ), ctypes.byref(nd), dims,
                                        ctypes.byref(nb)), "vox_gguf_tensor_info")
        return name.value.decode(), typ.value, list(dims)[:nd.value], nb.value

    def data(self, i: int) -> bytes:
        p = lib.vox_gguf_tensor_data(self.h, i)
        return ctypes.string_at(p, self.info(i)[3]) if p else b""

    def get_int(self, key: str) -> int:
        v = _I64()
        _check(lib.vox_gguf_get_int(self.h, key.encode(), ctypes.byref(v)), "vox_gguf_get_int")
        return v.value

    def get_float(self, key: str) -> float:
        v = ctypes.c_double()
        _check(lib.vox_gguf_get_float(self.h, key.encode(), ctypes.byref(v)), "vox_gguf_get_float")
        return v.value

    def get_string(self, key: str):
        v = lib.vox_gguf_get_string(self.h, key.encode())
        return None if v is None else v.decode()

    def upload_q4(self, i: int, scratch, packed, flags: int = VOX_PACK_PLAIN, stream=None):
        _check(lib.vox_gguf_upload_q4(self.h, i, ptr(scratch), scratch.numel() * scratch.element_size(), flags,
                                      ptr(packed), stream_ptr(stream)), "vox_gguf_upload_q4")
