"""Device-side state of the synthetic workloads, built through libvox.

Weights are drawn by :mod:`synth` (GGUF Q4_0 blocks), copied to the GPU and
repacked there by ``vox_q4_pack``; caches, activations and workspaces are
plain torch allocations.  The objects keep every tensor alive and expose the
``vox_decoder`` / ``vox_encoder`` descriptors of include/vox.h.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

import synth

from . import vox as V


def to_dev(a: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def bf16_dev(bits: np.ndarray, device) -> torch.Tensor:
    """bf16 bit patterns (uint16) -> device bfloat16 tensor with the same bits."""
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)


def pack_q4(qs: np.ndarray, d: np.ndarray, device, flags: int = V.VOX_PACK_PLAIN):
    """GGUF (qs, d) -> packed device weight; returns (tensor, vox_q4_weight)."""
    n, nb, _ = qs.shape
    k = nb * 32
    g = to_dev(synth.gguf_bytes(qs, d).reshape(-1), device)
    packed = torch.empty(V.vox_q4_packed_bytes(n, k), dtype=torch.uint8, device=device)
    V.vox_q4_pack(g, n, k, flags, packed)
    del g
    return packed, V.weight(packed, n, k)


def stack_rows(*parts):
    return (np.concatenate([p[0] for p in parts], axis=0), np.concatenate([p[1] for p in parts], axis=0))


def decoder_weights(shape: synth.DecoderShape, L: int, seed: int, device):
    """Packed weights of L decoder layers, the embedding and the LM head:
    (tensors to keep alive, [wqkv], [wo], [w13], [w2], embedding, lm_head)."""
    keep, wqkv, wo, w13, w2 = [], [], [], [], []
    for l in range(L):
        w = synth.decoder_layer_weights(shape, l, seed)
        for lst, (qs, d), flags in ((wqkv, stack_rows(w["wq"], w["wk"], w["wv"]), V.VOX_PACK_PLAIN),
                                    (wo, w["wo"], V.VOX_PACK_PLAIN),
                                    (w13, stack_rows(w["w1"], w["w3"]), V.VOX_PACK_GATE_UP),
                                    (w2, w["w2"], V.VOX_PACK_PLAIN)):
            t, desc = pack_q4(qs, d, device, flags)
            keep.append(t)
            lst.append(desc)
    emb_t, emb = pack_q4(*synth.q4_blocks(shape.vocab, shape.dim, seed, synth.EMB_ID), device)
    lm_t, lm = pack_q4(*synth.q4_blocks(shape.vocab, shape.dim, seed, synth.LM_HEAD_ID), device)
    keep += [emb_t, lm_t]
    return keep, wqkv, wo, w13, w2, emb, lm


class BatchDecoderModel:
    """n_seq independent sequences over the synthetic decoder, each with its
    own rolling cache in 64-slot pages of per-layer pools (synth.page_pool),
    assigned by synth.page_table.  positions[s] slots of sequence s are taken
    as present; the next step writes position positions[s]."""

    def __init__(self, shape: synth.DecoderShape, n_seq: int, positions, tokens, seed: int = 0, device="cuda",
                 n_layers=None, eps: float = 1e-5, window=None, spare_pages: int = 3, device_fill: bool = False,
                 rope_theta: float = 0.0):
        self.shape, self.seed, self.device = shape, seed, device
        self.L = shape.n_layers if n_layers is None else n_layers
        self.W = shape.window if window is None else window
        self.n_seq = n_seq
        pps = self.W // synth.PAGE_SLOTS
        self.n_pages = n_seq * pps + spare_pages
        D, F, QD, KVD = shape.dim, shape.ffn, shape.q_dim, shape.kv_dim
        keep, wqkv, wo, w13, w2, emb, lm = decoder_weights(shape, self.L, seed, device)
        self.k_pool, self.v_pool = [], []
        for l in range(self.L):
            if device_fill:
                # timing only: N(0,1) bf16 drawn on the device (seeded torch generator)
                gen = torch.Generator(device=device)
                shp = (self.n_pages, shape.n_kv_heads, synth.PAGE_SLOTS, shape.head_dim)
                for pools, off in ((self.k_pool, 0), (self.v_pool, 1)):
                    gen.manual_seed(seed * 1000 + 2 * l + off)
                    pools.append(torch.randn(shp, generator=gen, device=device).to(torch.bfloat16))
                continue
            kb, vb = synth.page_pool(shape, l, self.n_pages, seed)
            self.k_pool.append(bf16_dev(kb, device))
            self.v_pool.append(bf16_dev(vb, device))
        self.table_np = synth.page_table(n_seq, self.W, self.n_pages, seed)
        self.page_table = to_dev(self.table_np, device)
        self._keep = keep
        self.wqkv, self.wo, self.w13, self.w2 = wqkv, wo, w13, w2
        f32 = dict(dtype=torch.float32, device=device)
        self.token = torch.tensor(list(tokens), dtype=torch.int32, device=device)
        self.pos = torch.tensor(list(positions), dtype=torch.int64, device=device)
        self.x = torch.zeros(n_seq, D, **f32)
        self.h = torch.zeros(n_seq, D, **f32)
        self.qkv = torch.zeros(n_seq, QD + 2 * KVD, **f32)
        self.attn = torch.zeros(n_seq, QD, **f32)
        self.act = torch.zeros(n_seq, F, **f32)
        self.logits = torch.zeros(n_seq, shape.vocab, **f32)
        Arr = V.vox_q4_weight * self.L
        Ptr = ctypes.c_void_p * self.L
        self._arrs = [Arr(*wqkv), Arr(*wo), Arr(*w13), Arr(*w2), Ptr(*[t.data_ptr() for t in self.k_pool]),
                      Ptr(*[t.data_ptr() for t in self.v_pool])]
        b = V.vox_decoder_batch()
        d = b.d
        d.n_layers, d.dim, d.n_q_heads, d.n_kv_heads = self.L, D, shape.n_q_heads, shape.n_kv_heads
        d.head_dim, d.ffn, d.vocab, d.window, d.eps = shape.head_dim, F, shape.vocab, self.W, eps
        d.wqkv, d.wo, d.w13, d.w2 = [ctypes.cast(a, ctypes.POINTER(V.vox_q4_weight)) for a in self._arrs[:4]]
        d.embedding, d.lm_head = emb, lm
        d.k_cache = ctypes.cast(self._arrs[4], ctypes.POINTER(ctypes.c_void_p))
        d.v_cache = ctypes.cast(self._arrs[5], ctypes.POINTER(ctypes.c_void_p))
        for name in ("token", "pos", "x", "h", "qkv", "attn", "act", "logits"):
            setattr(d, name, getattr(self, name).data_ptr())
        d.rope_theta = rope_theta
        b.n_seq, b.n_pages, b.page_table = n_seq, self.n_pages, self.page_table.data_ptr()
        ws = V.vox_decoder_batch_workspace(b)
        self.workspace = torch.zeros(ws, dtype=torch.uint8, device=device)
        d.workspace, d.ws_bytes = self.workspace.data_ptr(), ws
        self.batch = b

    def step(self, stream=None):
        V.vox_decoder_batch_step(self.batch, stream)

    def capture(self):
        """CUDA graph of one batched step (one eager run on a side stream first)."""
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            self.step()
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.step()
        return g

    def weight_bytes(self) -> int:
        tot = sum(w.n * w.k * 18 // 32 for w in self.wqkv + self.wo + self.w13 + self.w2)
        return tot + self.shape.vocab * self.shape.dim * 18 // 32 + self.n_seq * self.shape.dim * 18 // 32

    def kv_bytes(self, positions) -> int:
        """bf16 K and V bytes the attention reads when sequence s has written positions[s]."""
        per = sum(min(p + 1, self.W) for p in positions)
        return self.L * 2 * self.shape.n_kv_heads * per * self.shape.head_dim * 2

    def launches(self) -> int:
        """Kernels one batched step launches: the embedding rows, per layer
        QKV, attention, combine, Wo, W1||W3 and W2, plus one bf16 cast before
        each of Wo and W2 where those run on the tcgen05 GEMM (from 4
        sequences on, unless VOX_BATCH_GEMM=0), then the LM head and the
        position advance."""
        sh = self.shape
        gemm = (self.n_seq >= 4 and not os.environ.get("VOX_BATCH_GEMM", "").startswith("0")
                and (sh.n_q_heads * sh.head_dim) % 64 == 0 and sh.ffn % 64 == 0)
        return 1 + self.L * (8 if gemm else 6) + 1 + 1


class DecoderModel:
    """26-layer synthetic decoder (or fewer layers) with rolling caches.

    ``filled`` positions 0..filled-1 are taken as already present in the
    caches (their contents are the seeded N(0,1) bf16 draws); the next step
    writes position ``filled``.
    """

    def __init__(self, shape: synth.DecoderShape, seed: int = 0, device="cuda", n_layers=None,
                 filled: int = 0, token: int = 0, eps: float = 1e-5, window=None, rope_theta: float = 0.0):
        self.shape = shape
        self.seed = seed
        self.device = device
        self.L = shape.n_layers if n_layers is None else n_layers
        self.W = shape.window if window is None else window
        self.eps = eps
        D, F = shape.dim, shape.ffn
        QD, KVD = shape.q_dim, shape.kv_dim
        keep = []
        wqkv, wo, w13, w2, kc, vc = [], [], [], [], [], []
        for l in range(self.L):
            w = synth.decoder_layer_weights(shape, l, seed)
            t, desc = pack_q4(*stack_rows(w["wq"], w["wk"], w["wv"]), device)
            keep.append(t); wqkv.append(desc)
            t, desc = pack_q4(*w["wo"], device)
            keep.append(t); wo.append(desc)
            t, desc = pack_q4(*stack_rows(w["w1"], w["w3"]), device, V.VOX_PACK_GATE_UP)
            keep.append(t); w13.append(desc)
            t, desc = pack_q4(*w["w2"], device)
            keep.append(t); w2.append(desc)
            kb, vb = synth.decoder_layer_cache(shape, l, seed, self.W)
            kt, vt = bf16_dev(kb, device), bf16_dev(vb, device)
            keep += [kt, vt]
            kc.append(kt.data_ptr()); vc.append(vt.data_ptr())
        self.emb_t, emb = pack_q4(*synth.q4_blocks(shape.vocab, D, seed, synth.EMB_ID), device)
        self.lm_t, lm = pack_q4(*synth.q4_blocks(shape.vocab, D, seed, synth.LM_HEAD_ID), device)
        self._keep = keep
        self.wqkv, self.wo, self.w13, self.w2 = wqkv, wo, w13, w2
        self.k_cache = [keep[6 * l + 4] for l in range(self.L)]
        self.v_cache = [keep[6 * l + 5] for l in range(self.L)]

        f32 = dict(dtype=torch.float32, device=device)
        self.token = torch.tensor([token], dtype=torch.int32, device=device)
        self.pos = torch.tensor([filled], dtype=torch.int64, device=device)
        self.x = torch.zeros(D, **f32)
        self.h = torch.zeros(D, **f32)
        self.qkv = torch.zeros(QD + 2 * KVD, **f32)
        self.attn = torch.zeros(QD, **f32)
        self.act = torch.zeros(F, **f32)
        self.logits = torch.zeros(shape.vocab, **f32)

        Arr = V.vox_q4_weight * self.L
        Ptr = ctypes.c_void_p * self.L
        self._arrs = [Arr(*wqkv), Arr(*wo), Arr(*w13), Arr(*w2), Ptr(*kc), Ptr(*vc)]
        dec = V.vox_decoder()
        dec.n_layers, dec.dim, dec.n_q_heads, dec.n_kv_heads = self.L, D, shape.n_q_heads, shape.n_kv_heads
        dec.head_dim, dec.ffn, dec.vocab, dec.window, dec.eps = shape.head_dim, F, shape.vocab, self.W, eps
        dec.rope_theta = rope_theta
        dec.wqkv, dec.wo, dec.w13, dec.w2 = [ctypes.cast(a, ctypes.POINTER(V.vox_q4_weight)) for a in self._arrs[:4]]
        dec.embedding, dec.lm_head = emb, lm
        dec.k_cache = ctypes.cast(self._arrs[4], ctypes.POINTER(ctypes.c_void_p))
        dec.v_cache = ctypes.cast(self._arrs[5], ctypes.POINTER(ctypes.c_void_p))
        for name in ("token", "pos", "x", "h", "qkv", "attn", "act", "logits"):
            setattr(dec, name, getattr(self, name).data_ptr())
        ws = V.vox_decoder_workspace(dec)
        self.workspace = torch.zeros(ws, dtype=torch.uint8, device=device)
        dec.workspace, dec.ws_bytes = self.workspace.data_ptr(), ws
        self.dec = dec
        self.emb, self.lm = emb, lm

    def step(self, stream=None):
        """One token step as one persistent launch (vox_decoder_step)."""
        V.vox_decoder_step(self.dec, stream)

    def step_kernels(self, stream=None):
        """The same step as the library's per-kernel launch sequence."""
        V.vox_decoder_step_kernels(self.dec, stream)

    def step_fused(self, stream=None):
        """The same step with the projections between attentions fused into
        persistent launches."""
        V.vox_decoder_step_fused(self.dec, stream)

    # ----------------------------------------------------------- graphs
    def capture(self, fn=None):
        """Capture `fn` (default: one decoder step) into a CUDA graph.  One
        eager run on a side stream first, as torch requires before capture."""
        fn = self.step if fn is None else fn
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            fn()
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        return g

    def gemv_chain(self):
        """The step's projections alone (same launches, weights and epilogues
        as vox_decoder_step, without attention): used to time the GEMV."""
        QD, KVD, D, F = self.shape.q_dim, self.shape.kv_dim, self.shape.dim, self.shape.ffn
        ws = self.workspace
        for l in range(self.L):
            e = V.vox_epilogue(op=V.VOX_EP_KV_APPEND, rmsnorm=1, eps=self.eps, k_cache=self.k_cache[l].data_ptr(),
                               v_cache=self.v_cache[l].data_ptr(), n_kv_heads=self.shape.n_kv_heads,
                               head_dim=self.shape.head_dim, window=self.W, q_rows=QD, pos_dev=self.pos.data_ptr())
            V.vox_q4_gemv(self.wqkv[l], self.x, 1, D, self.qkv, QD + 2 * KVD, e, ws, ws.numel())
            r = V.vox_epilogue(op=V.VOX_EP_RESIDUAL, residual=self.x.data_ptr(), ldr=D)
            V.vox_q4_gemv(self.wo[l], self.attn, 1, QD, self.h, D, r, ws, ws.numel())
            f = V.vox_epilogue(op=V.VOX_EP_SILU_MUL, rmsnorm=1, eps=self.eps)
            V.vox_q4_gemv(self.w13[l], self.h, 1, D, self.act, F, f, ws, ws.numel())
            r2 = V.vox_epilogue(op=V.VOX_EP_RESIDUAL, residual=self.h.data_ptr(), ldr=D)
            V.vox_q4_gemv(self.w2[l], self.act, 1, F, self.x, D, r2, ws, ws.numel())
        am = V.vox_epilogue(op=V.VOX_EP_ARGMAX, rmsnorm=1, eps=self.eps, argmax=self.token.data_ptr())
        V.vox_q4_gemv(self.lm, self.x, 1, D, self.logits, self.shape.vocab, am, ws, ws.numel())

    def gemv_chain_launches(self) -> int:
        return 4 * self.L + 1

    def gemv_chain_bytes(self) -> int:
        return sum(w.n * w.k * 18 // 32 for w in self.wqkv + self.wo + self.w13 + self.w2) + \
            self.shape.vocab * self.shape.dim * 18 // 32

    def attn_chain(self, pos: int):
        """The step's attention launches alone (per layer: split-KV + combine),
        at a host-given position."""
        wsb = V.vox_gqa_decode_attn_workspace(self.shape.n_q_heads, self.shape.n_kv_heads, self.shape.head_dim,
                                              self.W)
        ws = self.workspace[self.workspace.numel() - wsb:]
        for l in range(self.L):
            V.vox_gqa_decode_attn(self.qkv, self.k_cache[l], self.v_cache[l], self.attn, self.shape.n_q_heads,
                                  self.shape.n_kv_heads, self.shape.head_dim, self.W, pos,
                                  1.0 / self.shape.head_dim ** 0.5, ws, wsb)

    def step_launches(self) -> int:
        """Kernels one vox_decoder_step launches."""
        return 1

    def step_fused_launches(self) -> int:
        """Launches of one vox_decoder_step_fused: its own kernels."""
        return 1 + 3 * self.L

    def step_kernels_launches(self) -> int:
        """Kernels one vox_decoder_step_kernels launches."""
        return 1 + self.L * 6 + 1 + 1

    def weight_bytes(self) -> int:
        """Packed Q4 bytes streamed per step (all layers + LM head + one embedding row)."""
        tot = sum(w.n * w.k * 18 // 32 for w in self.wqkv + self.wo + self.w13 + self.w2)
        return tot + self.shape.vocab * self.shape.dim * 18 // 32 + self.shape.dim * 18 // 32

    def kv_bytes(self, pos: int) -> int:
        """bf16 K and V bytes the attention reads after position ``pos`` was written."""
        nv = min(pos + 1, self.W)
        return self.L * 2 * self.shape.n_kv_heads * nv * self.shape.head_dim * 2


class EncoderModel:
    """Synthetic encoder chunk: rows x dim input, per-layer history caches, adapter."""

    def __init__(self, shape: synth.EncoderShape, seed: int = 0, device="cuda", n_layers=None, eps: float = 1e-5,
                 tap: bool = False, stream: bool = False):
        self.shape = shape
        self.L = shape.n_layers if n_layers is None else n_layers
        D, F, R = shape.dim, shape.ffn, shape.rows
        keep = []
        wqkv, wo, wup, wdown, kh, vh = [], [], [], [], [], []
        for l in range(self.L):
            w = synth.encoder_layer_weights(shape, l, seed)
            for key, lst in (("wqkv", wqkv), ("wo", wo), ("wup", wup), ("wdown", wdown)):
                t, desc = pack_q4(*w[key], device)
                keep.append(t); lst.append(desc)
            kb, vb = synth.encoder_layer_history(shape, l, seed)
            kt, vt = bf16_dev(kb, device), bf16_dev(vb, device)
            keep += [kt, vt]
            kh.append(kt.data_ptr()); vh.append(vt.data_ptr())
        self.ad_t, ad = pack_q4(*synth.q4_blocks(shape.adapter_out, shape.downsample * D, seed, synth.ADAPTER_ID),
                                device)
        self.ad2_t, ad2 = pack_q4(*synth.q4_blocks(shape.adapter_out, shape.adapter_out, seed, synth.ADAPTER2_ID),
                                  device)
        self._keep = keep
        self.wqkv, self.wo, self.wup, self.wdown = wqkv, wo, wup, wdown
        self.k_hist = [keep[6 * l + 4] for l in range(self.L)]
        self.v_hist = [keep[6 * l + 5] for l in range(self.L)]
        self.x0 = to_dev(synth.activations(R, D, seed, synth.ENC_X_ID), device)
        self.x = self.x0.clone()
        bf = dict(dtype=torch.bfloat16, device=device)
        self.xn = torch.zeros(R, D, **bf)
        self.qkv = torch.zeros(R, 3 * D, **bf)
        self.att = torch.zeros(R, D, **bf)
        self.up = torch.zeros(R, F, **bf)
        self.mid = torch.zeros(R // shape.downsample, shape.adapter_out, **bf)
        self.out = torch.zeros(R // shape.downsample, shape.adapter_out, dtype=torch.float32, device=device)
        Arr = V.vox_q4_weight * self.L
        Ptr = ctypes.c_void_p * self.L
        self._arrs = [Arr(*wqkv), Arr(*wo), Arr(*wup), Arr(*wdown), Ptr(*kh), Ptr(*vh)]
        e = V.vox_encoder()
        e.n_layers, e.dim, e.n_heads, e.head_dim = self.L, D, shape.n_heads, shape.head_dim
        e.ffn, e.window, e.rows, e.adapter_out, e.eps = F, shape.window, R, shape.adapter_out, eps
        e.wqkv, e.wo, e.wup, e.wdown = [ctypes.cast(a, ctypes.POINTER(V.vox_q4_weight)) for a in self._arrs[:4]]
        e.adapter, e.adapter2 = ad, ad2
        e.adapter_mid = self.mid.data_ptr()
        e.k_hist = ctypes.cast(self._arrs[4], ctypes.POINTER(ctypes.c_void_p))
        e.v_hist = ctypes.cast(self._arrs[5], ctypes.POINTER(ctypes.c_void_p))
        for name in ("x", "xn", "qkv", "att", "up"):
            setattr(e, name, getattr(self, name).data_ptr())
        e.adapter_out_buf = self.out.data_ptr()
        # the last layer's input and mid-layer residual, for per-kernel checks of that layer
        self.tap = torch.zeros(2, R, D, dtype=torch.float32, device=device) if tap else None
        e.tap = self.tap.data_ptr() if tap else None
        self.enc = e
        self.adapter, self.adapter2 = ad, ad2
        # streaming: a second set of history buffers that receives the next chunk's history
        self.k_next = self.v_next = None
        if stream:
            self.k_next = [torch.zeros_like(t) for t in self.k_hist]
            self.v_next = [torch.zeros_like(t) for t in self.v_hist]
            self._point_history()

    def _point_history(self):
        Ptr = ctypes.c_void_p * self.L
        self._hist_arrs = [Ptr(*[t.data_ptr() for t in lst]) for lst in (self.k_hist, self.v_hist, self.k_next,
                                                                          self.v_next)]
        e = self.enc
        e.k_hist, e.v_hist, e.k_hist_next, e.v_hist_next = [ctypes.cast(a, ctypes.POINTER(ctypes.c_void_p))
                                                            for a in self._hist_arrs]

    def swap_history(self):
        """After a streamed chunk: the written next histories become the histories."""
        self.k_hist, self.k_next = self.k_next, self.k_hist
        self.v_hist, self.v_next = self.v_next, self.v_hist
        self._point_history()

    def set_input(self, x: np.ndarray):
        """A new chunk input (fp32 [rows][dim]); reset() restores it."""
        self.x0 = to_dev(x, self.x.device)
        self.x.copy_(self.x0)

    def reset(self):
        self.x.copy_(self.x0)

    def run(self, stream=None):
        V.vox_encoder_chunk(self.enc, stream)

    def gemm_flops(self) -> int:
        s = self.shape
        R, D, F = s.rows, s.dim, s.ffn
        per_layer = 2 * R * D * (3 * D + D + F) + 2 * R * F * D
        rd = R // s.downsample
        return self.L * per_layer + 2 * rd * (s.downsample * D) * s.adapter_out + 2 * rd * s.adapter_out ** 2
