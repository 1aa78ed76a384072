"""Small, self-contained launches of one kernel for an ncu capture.

    python -m bit_quantized_transformer_b200.profile_cases gemv N K [--launches L]
    python -m bit_quantized_transformer_b200.profile_cases attn POS [--launches L]
    python -m bit_quantized_transformer_b200.profile_cases gemm N K M [--launches L]

gemv: L launches of the Q4_0 GEMV (M = 1, no epilogue) on one packed N x K
      matrix (seeded synthetic weights as in the decoder workload).
attn: L launches of the split-KV decode attention on one decoder-shaped
      layer (32 query / 8 kv heads x 128, 8192-slot rolling cache, bf16)
      after position POS was written.
gemm: L launches of the Q4_0 GEMM (tcgen05) on one packed N x K matrix and
      M bf16 activation rows (bf16 output).
Each case holds well under 1 GB on the device and checks the device status
word at the end; it prints one line and exits 0.
"""
from __future__ import annotations

import argparse
import math
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def main(argv=None) -> int:
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("case", choices=["gemv", "attn", "gemm"])
    p.add_argument("args", type=int, nargs="+")
    p.add_argument("--launches", type=int, default=4)
    a = p.parse_args(argv)

    import torch

    import synth
    from bit_quantized_transformer_b200 import build

    build.build()
    from bit_quantized_transformer_b200 import vox as V
    from bit_quantized_transformer_b200 import workloads as WL

    if a.case == "gemv":
        n, k = a.args[0], a.args[1]
        qs, d = synth.q4_blocks(n, k, 0, 77)
        packed, w = WL.pack_q4(qs, d, "cuda")
        x = WL.to_dev(synth.activations(1, k, 0, 78), "cuda")
        y = torch.empty(1, n, device="cuda")
        wsb = V.vox_q4_gemv_workspace(w, 1, None)
        ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
        for _ in range(a.launches):
            V.vox_q4_gemv(w, x, 1, k, y, n, None, ws, wsb)
        what = f"gemv {n}x{k}: {packed.numel()} weight bytes per launch"
    elif a.case == "gemm":
        n, k, m = a.args[0], a.args[1], a.args[2]
        qs, d = synth.q4_blocks(n, k, 0, 79)
        packed, w = WL.pack_q4(qs, d, "cuda")
        x = WL.bf16_dev(synth.bf16_normal((m, k), 0, 80), "cuda")
        y = torch.empty(m, n, dtype=torch.bfloat16, device="cuda")
        for _ in range(a.launches):
            V.vox_q4_gemm(w, x, V.VOX_BF16, m, k, y, V.VOX_BF16, n)
        what = f"gemm {n}x{k} M={m}: {2 * m * n * k} flop per launch"
    else:
        pos = a.args[0]
        n_q, n_kv, hd, W = 32, 8, 128, 8192
        kc = torch.randn(n_kv, W, hd, device="cuda").to(torch.bfloat16)
        vc = torch.randn(n_kv, W, hd, device="cuda").to(torch.bfloat16)
        q = torch.randn(n_q, hd, device="cuda")
        out = torch.empty(n_q, hd, device="cuda")
        wsb = V.vox_gqa_decode_attn_workspace(n_q, n_kv, hd, W)
        ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
        for _ in range(a.launches):
            V.vox_gqa_decode_attn(q, kc, vc, out, n_q, n_kv, hd, W, pos, 1.0 / math.sqrt(hd), ws, wsb)
        what = f"attn pos {pos}: {2 * n_kv * min(pos + 1, W) * hd * 2} cache bytes per launch"
    torch.cuda.synchronize()
    assert V.vox_device_status(True) == 0
    print(f"ok {what} x {a.launches}")
    return 0


if __name__ == "__main__":
    sys.exit(main())
