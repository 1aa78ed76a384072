"""NumPy twin of the CPU oracle, plus the composed decoder / encoder references.

TEST INFRASTRUCTURE ONLY: only ``tests/``, ``__graft_entry__.smoke()`` and the
bench's CPU-baseline leg may import this module.  It shares no code with the
CUDA path and never imports it.  All arithmetic is float64 unless a step's
definition fixes another precision (bf16 storage of cache entries).

Two independent routes live here:

* the C oracle ``vox_ref.c`` (loaded through ctypes from ``libvoxref.so``,
  built by ``build_c()`` below with gcc), written as scalar loops;
* NumPy functions below, written independently with array operations and
  numpy/scipy library primitives (matmul, exp, erf).

The tests pin both against hand-built values and closed forms and check that
they agree with each other to 1e-12.

Definitions followed (page titles as on the pages):

* Q4_0: "Voxtral Mini 4B Realtime (Rust)", page 5 "Arquitetura" (GGUF Q4_0),
  w = (q - 8) * d with GGUF nibble order (reading R1).
* Decoder: "Mistral Voxtral Realtime 4B ... 순수 C 기반 CPU 전용 추론 구현",
  "모델 아키텍처": 26 layers, dim 3072, GQA 32/8; "주요 기능": rolling KV cache
  of 8192 positions.  Layer structure (pre-norm, RMSNorm eps 1e-5, SwiGLU FFN,
  no RoPE) is reading R3-R5; GQA mapping and 1/sqrt(head_dim) scale R7.
* Encoder: same page, "모델 아키텍처": 32 causal layers, dim 1280, 32 heads,
  window 750; adapter Linear(5120->3072) -> GELU -> Linear.  Ungated FFN with
  exact-erf GELU and RMSNorm is reading R8; history cache R9; downsample order
  R10.
* LM head + greedy argmax, lowest index on ties (R11).

One decoder layer and one encoder layer are pinned by closed forms of
special cases (zero or identity projections, a single visible key).  The
26-layer step and the 32-layer chunk as wholes are only the composition of
those pinned layers: beyond that they are parity unpinned (no published
logits exist).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libvoxref.so")
_lib = None

RMS_EPS = 1e-5   # reading R3


# ------------------------------------------------------------------ C oracle
def build_c(force: bool = False) -> str:
    """Compile vox_ref.c into libvoxref.so (gcc, OpenMP)."""
    src = os.path.join(_HERE, "vox_ref.c")
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(src):
        cmd = ["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared", "-o", _LIB_PATH, src, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB_PATH


def c_lib():
    global _lib
    if _lib is None:
        build_c()
        lib = ctypes.CDLL(_LIB_PATH)
        P, I64, D = ctypes.c_void_p, ctypes.c_int64, ctypes.c_double
        lib.vr_half_to_double.restype = D
        lib.vr_half_to_double.argtypes = [ctypes.c_uint16]
        lib.vr_bf16_to_double.restype = D
        lib.vr_bf16_to_double.argtypes = [ctypes.c_uint16]
        lib.vr_f32_to_bf16.restype = ctypes.c_uint16
        lib.vr_f32_to_bf16.argtypes = [ctypes.c_float]
        lib.vr_q4_row.argtypes = [P, P, I64, P]
        lib.vr_q4_dequant_f32.argtypes = [P, P, I64, I64, I64, I64, P]
        lib.vr_q4_dequant_bf16.argtypes = [P, P, I64, I64, I64, I64, P]
        lib.vr_q4_matvec.argtypes = [P, P, I64, I64, I64, I64, P, I64, I64, P]
        lib.vr_q4_matvec_blocksum.argtypes = [P, P, I64, I64, P, I64, I64, P]
        lib.vr_kv_slot.restype = I64
        lib.vr_kv_slot.argtypes = [I64, I64]
        lib.vr_kv_append.argtypes = [P, P, P, P, ctypes.c_int, ctypes.c_int, I64, I64]
        lib.vr_gqa_attn.argtypes = [P, P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int, I64, I64, D, P]
        _lib = lib
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def c_dequant_f32(qs, d, row0=0, nrows=None):
    n, nb, _ = qs.shape
    nrows = n - row0 if nrows is None else nrows
    out = np.empty((nrows, nb * 32), np.float32)
    c_lib().vr_q4_dequant_f32(_p(qs), _p(d), n, nb * 32, row0, nrows, _p(out))
    return out


def c_dequant_bf16(qs, d, row0=0, nrows=None):
    n, nb, _ = qs.shape
    nrows = n - row0 if nrows is None else nrows
    out = np.empty((nrows, nb * 32), np.uint16)
    c_lib().vr_q4_dequant_bf16(_p(qs), _p(d), n, nb * 32, row0, nrows, _p(out))
    return out


def c_matvec(qs, d, x, row0=0, nrows=None):
    """y[m, r] (float64) for output rows [row0, row0+nrows), dense route."""
    n, nb, _ = qs.shape
    x = np.ascontiguousarray(np.atleast_2d(x), dtype=np.float32)
    nrows = n - row0 if nrows is None else nrows
    y = np.empty((x.shape[0], nrows), np.float64)
    c_lib().vr_q4_matvec(_p(qs), _p(d), n, nb * 32, row0, nrows, _p(x), x.shape[0], x.shape[1], _p(y))
    return y


def c_matvec_blocksum(qs, d, x):
    n, nb, _ = qs.shape
    x = np.ascontiguousarray(np.atleast_2d(x), dtype=np.float32)
    y = np.empty((x.shape[0], n), np.float64)
    c_lib().vr_q4_matvec_blocksum(_p(qs), _p(d), n, nb * 32, _p(x), x.shape[0], x.shape[1], _p(y))
    return y


def c_kv_append(k_cache, v_cache, k_new, v_new, pos):
    n_kv, W, hd = k_cache.shape
    k_new = np.ascontiguousarray(k_new, np.float32)
    v_new = np.ascontiguousarray(v_new, np.float32)
    c_lib().vr_kv_append(_p(k_cache), _p(v_cache), _p(k_new), _p(v_new), n_kv, hd, W, pos)


def c_gqa_attn(q, k_cache, v_cache, pos, scale=None):
    n_kv, W, hd = k_cache.shape
    q = np.ascontiguousarray(q, np.float32)
    n_q = q.shape[0]
    scale = 1.0 / np.sqrt(hd) if scale is None else scale
    out = np.empty((n_q, hd), np.float64)
    c_lib().vr_gqa_attn(_p(q), _p(k_cache), _p(v_cache), n_q, n_kv, hd, W, pos, float(scale), _p(out))
    return out


# --------------------------------------------------------------- NumPy twin
def half_to_f64(d: np.ndarray) -> np.ndarray:
    """fp16 bit patterns -> float64 (numpy's cast serves as the library step)."""
    return np.asarray(d, np.uint16).view(np.float16).astype(np.float64)


def bf16_to_f64(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f32_to_bf16(f: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16, nearest-even, NaN -> 0x7FC0 (R2); array version."""
    u = np.ascontiguousarray(f, np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    nan = np.isnan(np.asarray(f, np.float32))
    r[nan] = 0x7FC0
    return r


def q4_codes(qs: np.ndarray) -> np.ndarray:
    """4-bit codes [n, nb, 32] in GGUF order: low nibbles first, then high (R1)."""
    return np.concatenate([qs & 0x0F, qs >> 4], axis=-1).astype(np.int64)


def q4_weights(qs: np.ndarray, d: np.ndarray) -> np.ndarray:
    """Exactly dequantised weights, float64 [n, k]."""
    n, nb, _ = qs.shape
    with np.errstate(invalid="ignore"):          # 0 * inf -> NaN is the defined result
        w = (q4_codes(qs) - 8).astype(np.float64) * half_to_f64(d)[:, :, None]
    return w.reshape(n, nb * 32)


def dequant_f32(qs, d):
    return q4_weights(qs, d).astype(np.float32)


def dequant_bf16(qs, d):
    return f32_to_bf16(dequant_f32(qs, d))


def matvec(qs, d, x):
    """Y[m, n] = sum_k w[n, k] x[m, k], float64."""
    return np.atleast_2d(np.asarray(x, np.float64)) @ q4_weights(qs, d).T


def rmsnorm(x, eps=RMS_EPS, g=None):
    """x / sqrt(mean(x^2) + eps) * g, per row, g = 1 by default (R3)."""
    x = np.asarray(x, np.float64)
    r = x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    return r if g is None else r * g


def silu(a):
    a = np.asarray(a, np.float64)
    return a / (1.0 + np.exp(-a))


def gelu(a):
    """Exact GELU: a * Phi(a) with the error function (R8)."""
    from scipy.special import erf

    a = np.asarray(a, np.float64)
    return 0.5 * a * (1.0 + erf(a / np.sqrt(2.0)))


def kv_slot(pos, window):
    return pos % window


def valid_slots(pos, window):
    """Number of valid slots after position ``pos`` was written (R6)."""
    return min(pos + 1, window)


def gqa_attn(q, k_cache, v_cache, pos, scale=None):
    """Array version of the rolling-window GQA decode attention (R6, R7)."""
    n_kv, W, hd = k_cache.shape
    q = np.asarray(q, np.float64)
    n_q = q.shape[0]
    scale = 1.0 / np.sqrt(hd) if scale is None else scale
    nv = valid_slots(pos, W)
    K = bf16_to_f64(k_cache[:, :nv, :])
    V = bf16_to_f64(v_cache[:, :nv, :])
    grp = n_q // n_kv
    out = np.empty((n_q, hd))
    for h in range(n_q):
        s = scale * (K[h // grp] @ q[h])
        p = np.exp(s - s.max())
        out[h] = (p / p.sum()) @ V[h // grp]
    return out


def attn_probs(q, k_cache, pos, scale=None):
    """Softmax probabilities [n_q, n_valid] (for the normalised error metric)."""
    n_kv, W, hd = k_cache.shape
    q = np.asarray(q, np.float64)
    scale = 1.0 / np.sqrt(hd) if scale is None else scale
    nv = valid_slots(pos, W)
    K = bf16_to_f64(k_cache[:, :nv, :])
    grp = q.shape[0] // n_kv
    P = np.empty((q.shape[0], nv))
    for h in range(q.shape[0]):
        s = scale * (K[h // grp] @ q[h])
        p = np.exp(s - s.max())
        P[h] = p / p.sum()
    return P


def split_partials(q, k_cache, v_cache, pos, n_split, scale=None):
    """Split-KV partials (m, l, o_unnormalised) over n_split contiguous slot ranges."""
    n_kv, W, hd = k_cache.shape
    q = np.asarray(q, np.float64)
    scale = 1.0 / np.sqrt(hd) if scale is None else scale
    nv = valid_slots(pos, W)
    bounds = np.linspace(0, nv, n_split + 1).astype(int)
    grp = q.shape[0] // n_kv
    parts = []
    for a, b in zip(bounds[:-1], bounds[1:]):
        ms, ls, os_ = [], [], []
        for h in range(q.shape[0]):
            if b <= a:
                ms.append(-np.inf); ls.append(0.0); os_.append(np.zeros(hd)); continue
            K = bf16_to_f64(k_cache[h // grp, a:b])
            V = bf16_to_f64(v_cache[h // grp, a:b])
            s = scale * (K @ q[h])
            m = s.max()
            p = np.exp(s - m)
            ms.append(m); ls.append(p.sum()); os_.append(p @ V)
        parts.append((np.array(ms), np.array(ls), np.array(os_)))
    return parts


def combine_partials(parts):
    """Log-sum-exp combine of split-KV partials."""
    M = np.max(np.stack([p[0] for p in parts]), axis=0)
    L = np.zeros_like(M)
    O = np.zeros_like(parts[0][2])
    for m, l, o in parts:
        w = np.where(np.isfinite(m), np.exp(m - M), 0.0)
        L += w * l
        O += w[:, None] * o
    return O / L[:, None]


def kv_append(k_cache, v_cache, k_new, v_new, pos):
    W = k_cache.shape[1]
    s = kv_slot(pos, W)
    k_cache[:, s, :] = f32_to_bf16(np.asarray(k_new, np.float32))
    v_cache[:, s, :] = f32_to_bf16(np.asarray(v_new, np.float32))


# ------------------------------------------------------------ paged caches
# Batched decode (voxtral.c page, "주요 기능": a rolling cache per stream and
# batched attention).  Reading R16: each sequence of a batch keeps its own
# rolling cache of W slots, stored in pages of PAGE_SLOTS consecutive slots
# of every kv head, drawn from a pool [n_pages][n_kv][PAGE_SLOTS][hd]; its
# table row names the page of each run of PAGE_SLOTS slots.  The paging only
# decides where a slot is stored: every sequence then follows the
# single-sequence definitions above unchanged.
PAGE_SLOTS = 64


def paged_to_cache(pool, table_row):
    """The logical rolling cache [n_kv][W][hd] (W = len(table_row) * 64) of
    one sequence: slot p is row p mod 64 of page table_row[p // 64]."""
    n_pages, n_kv, ps, hd = pool.shape
    W = len(table_row) * ps
    out = np.empty((n_kv, W, hd), pool.dtype)
    for c, page in enumerate(table_row):
        out[:, c * ps:(c + 1) * ps, :] = pool[page]
    return out


def paged_append(k_pool, v_pool, table_row, k_new, v_new, pos):
    """kv_append for a paged sequence: the slot pos mod W, in its page."""
    W = len(table_row) * PAGE_SLOTS
    s = kv_slot(pos, W)
    page, row = table_row[s // PAGE_SLOTS], s % PAGE_SLOTS
    k_pool[page, :, row, :] = f32_to_bf16(np.asarray(k_new, np.float32))
    v_pool[page, :, row, :] = f32_to_bf16(np.asarray(v_new, np.float32))


def argmax_lowest(v):
    """Greedy argmax, lowest index on ties (R11); numpy's argmax does this."""
    return int(np.argmax(np.asarray(v)))


# ----------------------------------------------------- normalised error (R13)
def gemv_error(y, y_ref, x, w):
    """max_{m,n} |y - y_ref| / (||x_m|| * ||w_n||)."""
    y = np.atleast_2d(np.asarray(y, np.float64))
    y_ref = np.atleast_2d(np.asarray(y_ref, np.float64))
    xn = np.linalg.norm(np.atleast_2d(np.asarray(x, np.float64)), axis=1)[:, None]
    wn = np.linalg.norm(np.asarray(w, np.float64), axis=1)[None, :]
    den = np.maximum(xn * wn, 1e-300)
    return float(np.max(np.abs(y - y_ref) / den))


def attn_error(o, o_ref, probs, v_cache_valid_f64, group):
    """max_{h,c} |o - o_ref| / (||p_h|| * ||V[:, c]||) for the head's kv group."""
    o = np.asarray(o, np.float64)
    err = 0.0
    for h in range(o.shape[0]):
        V = v_cache_valid_f64[h // group]          # [n_valid, hd]
        den = np.linalg.norm(probs[h]) * np.linalg.norm(V, axis=0)
        err = max(err, float(np.max(np.abs(o[h] - o_ref[h]) / np.maximum(den, 1e-300))))
    return err


# ------------------------------------------------------- composed references
def rope(x, pos, theta, head_dim):
    """Rotary position embedding of a vector of heads x [n_heads * head_dim]
    at position ``pos`` (reading R17; the pages do not mention positional
    encoding, so the decoder runs without it by default, reading R5): within
    each head the pair (x[2i], x[2i+1]) is rotated by the angle
    pos * theta^(-2i / head_dim), i = 0 .. head_dim/2 - 1.  theta <= 0: x unchanged."""
    x = np.asarray(x, np.float64)
    if theta <= 0:
        return x.copy()
    y = x.reshape(-1, head_dim).copy()
    i = np.arange(head_dim // 2)
    ang = pos * np.power(float(theta), -2.0 * i / head_dim)
    c, s = np.cos(ang), np.sin(ang)
    a, b = y[:, 0::2].copy(), y[:, 1::2].copy()
    y[:, 0::2] = a * c - b * s
    y[:, 1::2] = a * s + b * c
    return y.reshape(x.shape)


def decoder_layer(x, Wd, k_cache, v_cache, pos, n_q_heads, n_kv_heads, eps=RMS_EPS, rope_theta=0.0):
    """One pre-norm decoder layer at M=1 (readings R4-R7; optional RoPE R17).

    ``Wd`` maps names to dense float64 weight matrices (wq, wk, wv, wo, w1,
    w3, w2).  The caches are updated in place (bf16 storage of the new k, v,
    rounded from float32 as the stored format requires).  Returns a dict of
    all intermediates.
    """
    x = np.asarray(x, np.float64)
    n = rmsnorm(x, eps)
    hd = k_cache.shape[2]
    q = rope(Wd["wq"] @ n, pos, rope_theta, hd)
    k = rope(Wd["wk"] @ n, pos, rope_theta, hd)
    v = Wd["wv"] @ n
    kv_append(k_cache, v_cache, k.reshape(n_kv_heads, hd), v.reshape(n_kv_heads, hd), pos)
    o = gqa_attn(q.reshape(n_q_heads, hd), k_cache, v_cache, pos).reshape(-1)
    h = x + Wd["wo"] @ o
    n2 = rmsnorm(h, eps)
    a = silu(Wd["w1"] @ n2) * (Wd["w3"] @ n2)
    out = h + Wd["w2"] @ a
    return {"n": n, "q": q, "k": k, "v": v, "o": o, "h": h, "n2": n2, "a": a, "out": out}


def window_attn(Q, K, V, q_pos0, window, n_heads, head_dim, scale=None):
    """Causal sliding-window MHA: query i (absolute position q_pos0 + i) sees
    key j (absolute position j) iff pos_i - window < j <= pos_i (R8)."""
    Q = np.asarray(Q, np.float64)
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    scale = 1.0 / np.sqrt(head_dim) if scale is None else scale
    nq = Q.shape[0]
    out = np.zeros((nq, n_heads * head_dim))
    for i in range(nq):
        p = q_pos0 + i
        lo, hi = max(0, p - window + 1), p + 1
        for h in range(n_heads):
            sl = slice(h * head_dim, (h + 1) * head_dim)
            s = scale * (K[lo:hi, sl] @ Q[i, sl])
            e = np.exp(s - s.max())
            out[i, sl] = (e / e.sum()) @ V[lo:hi, sl]
    return out


def roll_history(hist, new, window):
    """Streaming chunks (voxtral.c page, "주요 기능": the encoder takes the audio
    in overlapping chunks; reading R18): the next chunk's history of a layer
    is the last `window` rows of this chunk's history followed by its own new
    k (or v) rows, oldest first."""
    both = np.concatenate([np.asarray(hist), np.asarray(new)], axis=0)
    return both[both.shape[0] - window:].copy()


def encoder_layer(X, Wd, k_hist, v_hist, window, n_heads, head_dim, eps=RMS_EPS):
    """One pre-norm encoder layer over a chunk of rows (R8, R9).

    ``k_hist``/``v_hist`` are float64 [n_hist, dim] (history rows at absolute
    positions 0..n_hist-1); the chunk rows sit at positions n_hist... .
    """
    X = np.asarray(X, np.float64)
    D = X.shape[1]
    n = rmsnorm(X, eps)
    qkv = n @ Wd["wqkv"].T
    q, k, v = qkv[:, :D], qkv[:, D:2 * D], qkv[:, 2 * D:]
    K = np.concatenate([k_hist, k], axis=0)
    V = np.concatenate([v_hist, v], axis=0)
    att = window_attn(q, K, V, k_hist.shape[0], window, n_heads, head_dim)
    h = X + att @ Wd["wo"].T
    u = gelu(rmsnorm(h, eps) @ Wd["wup"].T)
    return h + u @ Wd["wdown"].T


def adapter(Xd, W1, W2):
    """The audio-to-decoder adapter on downsampled rows: Linear(5120 -> 3072),
    exact-erf GELU, Linear(3072 -> 3072), no biases ("Mistral Voxtral Realtime
    4B ... 순수 C 기반 CPU 전용 추론 구현", "모델 아키텍처": adapter
    Linear -> GELU -> Linear; GELU form and no bias are readings R8)."""
    Xd = np.asarray(Xd, np.float64)
    return gelu(Xd @ np.asarray(W1, np.float64).T) @ np.asarray(W2, np.float64).T


def downsample_rows(X, factor=4):
    """Conv-4x downsample as a reshape: rows factor*r .. factor*r+factor-1
    concatenated in order form row r (R10)."""
    X = np.asarray(X)
    return X.reshape(X.shape[0] // factor, factor * X.shape[1])
