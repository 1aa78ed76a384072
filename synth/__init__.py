"""Seeded synthetic inputs, shared by the tests, the bench and the oracle runs.

This module holds none of the method's arithmetic. It only draws random
numbers and lays them out in the formats the method consumes:

* Q4_0 weights as the GGUF file format stores them: per block of 32 weights a
  little-endian fp16 scale ``d`` followed by 16 bytes of packed nibbles
  ("Voxtral Mini 4B Realtime (Rust)", page 5 "Arquitetura": GGUF Q4_0 path).
  The nibble bytes are uniform over 0..255, so each nibble is uniform 0..15;
  ``d = |N(0,1)| * 0.002`` rounded to fp16 by numpy.
* fp32 activations ~ N(0, 1).
* bf16 cache contents: N(0, 1) fp32 values cast to bf16 by torch's CPU cast.

Every tensor is drawn from ``numpy.random.default_rng([seed, tensor_id])``
with a fixed ``tensor_id`` enumeration, so any tensor of any workload can be
regenerated alone (the full-size parity tests regenerate single layers).
"""
from __future__ import annotations

import numpy as np

# ---------------------------------------------------------------- tensor ids
# decoder layer l uses ids 16*l + {WQ..VCACHE}
WQ, WK, WV, WO, W1, W3, W2, KCACHE, VCACHE, QVEC, KVEC, VVEC = range(12)
DEC_STRIDE = 16
EMB_ID = 1_000_000          # token embedding table, Q4_0 131072 x 3072
LM_HEAD_ID = 1_000_001      # LM head, Q4_0 131072 x 3072 (untied)
X_ID = 1_000_002            # decoder input / GEMV activation
TOKEN_ID = 1_000_003
# encoder layer l uses ids ENC_BASE + 16*l + {E_QKV..E_VHIST}
ENC_BASE = 2_000_000
E_QKV, E_O, E_UP, E_DOWN, E_KHIST, E_VHIST = range(6)
ADAPTER_ID = 3_000_000      # adapter first Linear, Q4_0 3072 x 5120
ENC_X_ID = 3_000_001        # encoder chunk input rows
ADAPTER2_ID = 3_000_002     # adapter second Linear, Q4_0 3072 x 3072
SWEEP_BASE = 4_000_000      # batched-shape sweep tensors
# batched decode: layer l's page pools use ids BATCH_BASE + 16*l + {0: K, 1: V}
BATCH_BASE = 5_000_000
BATCH_TABLE_ID = 5_999_999  # page assignment of the batch's sequences

D_SCALE = 0.002


def rng_for(seed: int, tensor_id: int) -> np.random.Generator:
    return np.random.default_rng([int(seed), int(tensor_id)])


def q4_blocks(n: int, k: int, seed: int, tensor_id: int):
    """Random Q4_0 weight of n rows x k columns (k a multiple of 32).

    Returns ``(qs, d)``: ``qs`` uint8 [n, k/32, 16] (the 16 nibble bytes of
    each block, GGUF byte order) and ``d`` uint16 [n, k/32] (fp16 bit
    patterns of the block scales).
    """
    if k % 32:
        raise ValueError("Q4_0 needs k % 32 == 0")
    rng = rng_for(seed, tensor_id)
    nb = k // 32
    qs = rng.integers(0, 256, size=n * nb * 16, dtype=np.uint8).reshape(n, nb, 16)
    d = (np.abs(rng.standard_normal(n * nb)) * D_SCALE).astype(np.float16)
    return qs, d.view(np.uint16).reshape(n, nb)


def gguf_bytes(qs: np.ndarray, d: np.ndarray) -> np.ndarray:
    """Interleave (qs, d) into the GGUF Q4_0 on-disk layout: uint8 [n, k/32, 18]."""
    n, nb, _ = qs.shape
    out = np.empty((n, nb, 18), dtype=np.uint8)
    out[:, :, 0:2] = d.astype("<u2").view(np.uint8).reshape(n, nb, 2)
    out[:, :, 2:18] = qs
    return out


def split_gguf(blocks: np.ndarray):
    """Inverse of :func:`gguf_bytes`."""
    n, nb, _ = blocks.shape
    d = np.ascontiguousarray(blocks[:, :, 0:2]).view("<u2").reshape(n, nb).astype(np.uint16)
    qs = np.ascontiguousarray(blocks[:, :, 2:18])
    return qs, d


def activations(m: int, k: int, seed: int, tensor_id: int) -> np.ndarray:
    """fp32 [m, k] ~ N(0, 1)."""
    return rng_for(seed, tensor_id).standard_normal((m, k)).astype(np.float32)


def bf16_normal(shape, seed: int, tensor_id: int) -> np.ndarray:
    """bf16 bit patterns (uint16) of N(0, 1) draws, cast by torch's CPU cast."""
    import torch

    f = rng_for(seed, tensor_id).standard_normal(int(np.prod(shape))).astype(np.float32)
    t = torch.from_numpy(f).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).reshape(shape)


def fp16_bits(values) -> np.ndarray:
    """fp16 bit patterns of the given values (numpy's cast)."""
    return np.asarray(values, dtype=np.float64).astype(np.float16).view(np.uint16)


# --------------------------------------------------------------- workloads
class DecoderShape:
    """Decoder of "Voxtral Mini 4B Realtime": 26 layers, dim 3072, GQA 32 query
    / 8 KV heads, head_dim 128, gated FFN 9216, vocab 131072, rolling window 8192
    (voxtral.c page, "모델 아키텍처" and "주요 기능")."""

    def __init__(self, n_layers=26, dim=3072, n_q_heads=32, n_kv_heads=8,
                 head_dim=128, ffn=9216, vocab=131072, window=8192):
        self.n_layers, self.dim = n_layers, dim
        self.n_q_heads, self.n_kv_heads, self.head_dim = n_q_heads, n_kv_heads, head_dim
        self.ffn, self.vocab, self.window = ffn, vocab, window

    @property
    def q_dim(self):
        return self.n_q_heads * self.head_dim

    @property
    def kv_dim(self):
        return self.n_kv_heads * self.head_dim


def decoder_layer_weights(shape: DecoderShape, layer: int, seed: int = 0):
    """GGUF-layout (qs, d) pairs for one decoder layer, keyed by name."""
    base = DEC_STRIDE * layer
    D, F = shape.dim, shape.ffn
    return {
        "wq": q4_blocks(shape.q_dim, D, seed, base + WQ),
        "wk": q4_blocks(shape.kv_dim, D, seed, base + WK),
        "wv": q4_blocks(shape.kv_dim, D, seed, base + WV),
        "wo": q4_blocks(D, shape.q_dim, seed, base + WO),
        "w1": q4_blocks(F, D, seed, base + W1),
        "w3": q4_blocks(F, D, seed, base + W3),
        "w2": q4_blocks(D, F, seed, base + W2),
    }


def decoder_layer_cache(shape: DecoderShape, layer: int, seed: int = 0, window=None):
    """bf16 K and V caches [n_kv_heads, window, head_dim] for one layer."""
    W = shape.window if window is None else window
    base = DEC_STRIDE * layer
    shp = (shape.n_kv_heads, W, shape.head_dim)
    return bf16_normal(shp, seed, base + KCACHE), bf16_normal(shp, seed, base + VCACHE)


class EncoderShape:
    """Audio encoder: 32 causal layers, dim 1280, 32 heads x 40, window 750,
    FFN 1280->5120->1280; adapter Linear 5120->3072 after a 4x downsample
    (voxtral.c page, "모델 아키텍처"; Rust page 5 "Arquitetura")."""

    def __init__(self, n_layers=32, dim=1280, n_heads=32, head_dim=40, ffn=5120,
                 window=750, rows=256, adapter_out=3072, downsample=4):
        self.n_layers, self.dim, self.n_heads, self.head_dim = n_layers, dim, n_heads, head_dim
        self.ffn, self.window, self.rows = ffn, window, rows
        self.adapter_out, self.downsample = adapter_out, downsample


def encoder_layer_weights(shape: EncoderShape, layer: int, seed: int = 0):
    base = ENC_BASE + DEC_STRIDE * layer
    D, F = shape.dim, shape.ffn
    return {
        "wqkv": q4_blocks(3 * D, D, seed, base + E_QKV),
        "wo": q4_blocks(D, D, seed, base + E_O),
        "wup": q4_blocks(F, D, seed, base + E_UP),
        "wdown": q4_blocks(D, F, seed, base + E_DOWN),
    }


def encoder_layer_history(shape: EncoderShape, layer: int, seed: int = 0):
    """bf16 K and V history rows [window, dim] (positions 0..window-1)."""
    base = ENC_BASE + DEC_STRIDE * layer
    shp = (shape.window, shape.dim)
    return bf16_normal(shp, seed, base + E_KHIST), bf16_normal(shp, seed, base + E_VHIST)


# --------------------------------------------------------- batched decode
PAGE_SLOTS = 64


def page_pool(shape: DecoderShape, layer: int, n_pages: int, seed: int = 0):
    """bf16 K and V page pools [n_pages, n_kv_heads, 64, head_dim] of one layer."""
    base = BATCH_BASE + DEC_STRIDE * layer
    shp = (n_pages, shape.n_kv_heads, PAGE_SLOTS, shape.head_dim)
    return bf16_normal(shp, seed, base), bf16_normal(shp, seed, base + 1)


def page_table(n_seq: int, window: int, n_pages: int, seed: int = 0) -> np.ndarray:
    """int32 [n_seq, window / 64]: distinct pages in a random order (every
    sequence owns window / 64 pages of the pool)."""
    pps = window // PAGE_SLOTS
    if n_seq * pps > n_pages:
        raise ValueError("pool too small for the batch")
    perm = rng_for(seed, BATCH_TABLE_ID).permutation(n_pages)[:n_seq * pps]
    return perm.astype(np.int32).reshape(n_seq, pps)
