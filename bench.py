#!/usr/bin/env python
"""Benchmark of the Q4_0 decode hot path on B200: prints ONE JSON line.

Workload (default, N=1): the full synthetic 26-layer decoder token step of
Voxtral Mini 4B Realtime (dim 3072, GQA 32/8, FFN 9216, Q4_0 weights, 131072 x
3072 LM head and embedding), rolling KV cache of 8192 positions filled to
8192 + 300 (wrapped), M = 1.  One step = one replay of the captured
vox_decoder_step graph: embedding row, 26 x (RMSNorm+QKV GEMV+rolling append,
split-KV GQA attention, Wo GEMV+residual, RMSNorm+W1||W3 GEMV+SiLU*mul, W2
GEMV+residual), RMSNorm+LM-head GEMV+argmax, position advance.  Every step
streams 2.8 GB (> 126 MB L2), so no flush is needed between steps.

value      = algorithmic bytes of all steps of all ranks / max-over-ranks time (GB/s)
ms_per_step= the decoder ms/step
roofline   = the dominant kernel (the Q4_0 GEMV, ~69% of the step's bytes),
             timed inside this run over the step's own 105 GEMV launches
e2e        = the same metric through the Python API with the token copied
             host->device before and device->host after every step
             (e2e_eager: the same with the C ABI's step called every step,
             no graph)
cpu_baseline / --impl reference = the CPU oracle (oracle/) on the host cores

Multi-GPU: one process per GPU (torchrun), independent replicas (the path
does not shard), barrier + max-over-ranks device time; "scaling": "weak".
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "Q4_0 GEMV weight GB/s (% of HBM peak); 26-layer decoder ms/step on 1 B200"
UNIT = "GB/s"
FALLBACK_HBM_GBS = 6650.0
FILLED = 8192 + 300
# dram bytes (read + write) per launch of the dominant kernel (the persistent
# step) from an ncu capture of the current kernel (profiles/); None until the
# kernel as it stands has been captured
STEP_TRAFFIC_BYTES_PER_LAUNCH = None
# the same for the per-projection GEMV (K1), from ncu captures of each decoder
# shape weighted by the step's launch mix (profiles/q4_gemv_lm_head_131072x3072.md);
# None: the kernel was split into per-epilogue instances after the last capture
GEMV_TRAFFIC_BYTES_PER_LAUNCH = None


def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=2000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=15.0, help="oracle sample budget")
    p.add_argument("--workload", choices=["decoder", "gemv", "layer", "encoder", "sweep", "kernel", "batch"],
                   default="decoder",
                   help="decoder: the headline line (default); gemv: the single 4096x3072 GEMV; layer: one "
                        "decoder layer at KV 1024; encoder: the 32-layer encoder chunk at M=256 "
                        "and its GEMMs; sweep: the decoder shapes at M in {1,4,16,64,256} and the attention at "
                        "KV in {512, 4096, 8192 wrapped}; kernel: a few launches of one kernel on one small "
                        "case (--kernel, --shape, --launches), sized for an ncu capture; batch: --seqs "
                        "sequences stepped together over paged caches (26 layers, KV 8192 wrapped)")
    p.add_argument("--seqs", type=int, default=8, help="batch workload: sequences (1..8)")
    p.add_argument("--kernel", choices=["gemv", "attn", "gemm", "step", "stepk", "encoder"], default="gemv",
                   help="kernel workload: gemv N K (M = 1), attn POS (decoder-shaped layer), gemm N K M, "
                        "step L (the persistent decoder step with L full-size layers, KV 8192 wrapped), "
                        "stepk L (the same step as the kernel sequence, eager), encoder L (the encoder chunk "
                        "with L layers and the adapter, eager)")
    p.add_argument("--shape", type=int, nargs="*", default=None)
    p.add_argument("--launches", type=int, default=4)
    return p.parse_args(argv)


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs)"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback 6.65 TB/s"


# ------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock and throttle reasons of this rank's GPU, read through NVML
    (read-only queries) every `period_s` by a background thread during the
    timed region; short regions still get samples."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))

    def __init__(self, torch_device: int, period_s: float = 0.002):
        self.dev = torch_device
        self.period = period_s
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self.err = None
        self._stop = None
        self._thr = None

    def _handle(self, nv):
        import torch

        try:
            uuid = str(torch.cuda.get_device_properties(self.dev).uuid)
            return nv.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:
            return nv.nvmlDeviceGetHandleByIndex(self.dev)

    def start(self):
        import threading

        try:
            import pynvml as nv

            nv.nvmlInit()
            h = self._handle(nv)
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            masks = [(name, getattr(nv, attr)) for name, attr in self.REASONS]
        except Exception as e:                       # no NVML: report it, time anyway
            self.err = f"nvml unavailable: {e}"
            return
        self._stop = threading.Event()

        def loop():
            while not self._stop.is_set():
                try:
                    self.samples.append(float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)))
                    r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                    for name, m in masks:
                        if r & m:
                            self.reasons.add(name)
                except Exception as e:
                    self.err = str(e)
                    return
                self._stop.wait(self.period)

        self._thr = threading.Thread(target=loop, daemon=True)
        self._thr.start()

    def stop(self):
        if self._thr is not None:
            self._stop.set()
            self._thr.join(timeout=5)
        out = {"sm_mhz": statistics.median(self.samples) if self.samples else None, "sm_max_mhz": self.max_mhz,
               "reasons": sorted(self.reasons), "samples": len(self.samples), "source": "nvml, 2 ms period"}
        if self.err:
            out["error"] = self.err
        return out


# ------------------------------------------------------- distributed
def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("LOCAL_RANK", "0"))


def dist_init(world, backend):
    import datetime

    import torch.distributed as dist

    if world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=300))


def aggregate(local_ms: float, steps: int, bytes_per_step: int, world: int):
    """Max-over-ranks time and the whole-job throughput (GB/s) of `world`
    independent replicas that each ran `steps` steps."""
    import torch
    import torch.distributed as dist

    t = torch.tensor([local_ms], dtype=torch.float64)
    if world > 1 and dist.is_initialized():
        if dist.get_backend() == "nccl":
            t = t.cuda()
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    max_ms = float(t.item())
    value = world * steps * bytes_per_step / (max_ms / 1e3) / 1e9
    return max_ms, value


def barrier(world):
    import torch.distributed as dist

    if world > 1 and dist.is_initialized():
        dist.barrier()


# ------------------------------------------------------------ timing
def time_replays(g, n, world):
    import torch

    barrier(world)
    torch.cuda.synchronize()
    s = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for _ in range(n):
        g.replay()
    e1.record(s)
    torch.cuda.synchronize()
    barrier(world)
    return e0.elapsed_time(e1)


# ------------------------------------------------------- CPU oracle
def oracle_decoder_sample(budget_s: float, layers=None, filled=FILLED):
    """The oracle's decoder layer (C oracle matvec + attention, numpy norms) on
    the first `layers` (default 4) layers of the same workload, cycled until
    `budget_s` of CPU time is spent.  Returns (bytes processed, seconds,
    layers done, threads)."""
    import numpy as np

    import synth
    from oracle import ref

    shape = synth.DecoderShape()
    D, QD, KVD = shape.dim, shape.q_dim, shape.kv_dim
    done, t_tot, bytes_tot = 0, 0.0, 0
    x = synth.activations(1, D, 0, synth.X_ID)[0]
    nl = 4 if layers is None else layers
    cached = [(synth.decoder_layer_weights(shape, l, 0), synth.decoder_layer_cache(shape, l, 0)) for l in range(nl)]
    while t_tot < budget_s:
        w, (kc, vc) = cached[done % nl]
        t0 = time.perf_counter()
        n = ref.rmsnorm(x).astype(np.float32)
        qkv = np.concatenate([ref.c_matvec(*w[k], n)[0] for k in ("wq", "wk", "wv")])
        ref.c_kv_append(kc, vc, qkv[QD:QD + KVD].reshape(shape.n_kv_heads, -1),
                        qkv[QD + KVD:].reshape(shape.n_kv_heads, -1), filled)
        o = ref.c_gqa_attn(qkv[:QD].reshape(shape.n_q_heads, -1).astype(np.float32), kc, vc, filled).reshape(-1)
        h = x + ref.c_matvec(*w["wo"], o.astype(np.float32))[0]
        n2 = ref.rmsnorm(h).astype(np.float32)
        a = ref.silu(ref.c_matvec(*w["w1"], n2)[0]) * ref.c_matvec(*w["w3"], n2)[0]
        x = (h + ref.c_matvec(*w["w2"], a.astype(np.float32))[0]).astype(np.float32)
        t_tot += time.perf_counter() - t0
        done += 1
        nw = sum(v[0].shape[0] * v[0].shape[1] * 32 for v in w.values())
        bytes_tot += nw * 18 // 32 + 2 * shape.n_kv_heads * min(filled + 1, shape.window) * shape.head_dim * 2
    threads = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return bytes_tot, t_tot, done, threads


def cpu_baseline(budget_s):
    b, t, n, threads = oracle_decoder_sample(budget_s)
    return {"value": b / t / 1e9, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{n} decoder-layer passes (the workload's first 4 layers, cycled; fp64 C oracle, "
                      f"OpenMP over rows), {b / 1e6:.1f} MB in {t:.1f} s"}


def run_reference(args):
    """The oracle on the host cores, timed as the reference arm."""
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    budget = max(0.05, 90.0 / max(1, args.steps + args.warmup))
    import numpy as np

    import synth
    from oracle import ref

    shape = synth.DecoderShape()
    w = synth.decoder_layer_weights(shape, 0, 0)
    kc, vc = synth.decoder_layer_cache(shape, 0, 0)
    x = synth.activations(1, shape.dim, 0, synth.X_ID)[0]
    mats = [w[k] for k in ("wq", "wk", "wv", "wo", "w1", "w3", "w2")]
    # calibrate rows per step so one step takes about `budget` seconds
    t0 = time.perf_counter()
    ref.c_matvec(*w["w1"], ref.rmsnorm(x).astype(np.float32), row0=0, nrows=512)
    per_row = (time.perf_counter() - t0) / 512
    rows = int(max(16, min(9216, budget / max(per_row, 1e-9))))
    tot_bytes, tot_t = 0, 0.0
    xin = {3072: ref.rmsnorm(x).astype(np.float32), 4096: synth.activations(1, 4096, 0, 1)[0],
           9216: synth.activations(1, 9216, 0, 2)[0]}
    for it in range(args.warmup + args.steps):
        qs, d = mats[it % len(mats)]
        r0 = (it * rows) % max(1, qs.shape[0] - rows + 1)
        nr = min(rows, qs.shape[0])
        t0 = time.perf_counter()
        ref.c_matvec(qs, d, xin[qs.shape[1] * 32], row0=r0, nrows=nr)
        dt = time.perf_counter() - t0
        if it >= args.warmup:
            tot_t += dt
            tot_bytes += nr * qs.shape[1] * 18
    value = tot_bytes / tot_t / 1e9
    threads = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    sample = f"per step {rows} rows of one decoder projection ({rows * 3072 * 18 // 32 / 1e6:.2f} MB Q4_0), fp64 C oracle"
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": tot_t / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": decoder_config(shape, world),
            "impl": "reference",
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------- ours
def try_graph(fn):
    """Capture fn into a CUDA graph (after one warm-up call on a side stream);
    None if the runtime refuses the capture."""
    import torch

    try:
        return graph_of(fn)
    except Exception:
        torch.cuda.synchronize()
        return None


def time_fn(fn, n, world, stream=None):
    """Device time of n calls of fn on the current stream, bracketed by a
    barrier and a synchronize on both sides (CUDA events on the launching
    stream)."""
    import torch

    barrier(world)
    torch.cuda.synchronize()
    s = torch.cuda.current_stream() if stream is None else stream
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for _ in range(n):
        fn()
    e1.record(s)
    torch.cuda.synchronize()
    barrier(world)
    return e0.elapsed_time(e1)


def run_ours(args):
    import torch

    rank, world, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        dist_init(world, "nccl")
    from bit_quantized_transformer_b200 import build

    if rank == 0 or not os.path.exists(build.LIB):
        build.build()
    barrier(world)
    import synth
    from bit_quantized_transformer_b200 import vox as V
    from bit_quantized_transformer_b200 import workloads as WL

    shape = synth.DecoderShape()
    dm = WL.DecoderModel(shape, seed=0, filled=FILLED, token=17)
    step_bytes = dm.weight_bytes() + dm.kv_bytes(FILLED)
    assert step_bytes == sum(decoder_bytes(shape))
    peak, peak_src = measured_peaks()

    # The three forms of the product's token step: one persistent launch
    # (vox_decoder_step), the per-kernel launch sequence
    # (vox_decoder_step_kernels) and persistent projection segments between
    # attention launches (vox_decoder_step_fused), each replayed from a CUDA
    # graph (launched directly if the runtime will not capture it).  All are
    # timed briefly; the fastest one is the headline.
    g_p = try_graph(dm.step)
    step_p = g_p.replay if g_p is not None else dm.step
    g_f = try_graph(dm.step_fused)
    step_f = g_f.replay if g_f is not None else dm.step_fused
    g_k = dm.capture(dm.step_kernels)
    forms = {}
    for name, fn in (("persistent", step_p), ("kernels", g_k.replay), ("fused", step_f)):
        for _ in range(max(3, args.warmup)):
            fn()
        torch.cuda.synchronize()
        assert V.vox_device_status(True) == 0, f"device status after the {name} warm-up"
        forms[name] = time_fn(fn, 10, world) / 10
    form = min(forms, key=forms.get)
    step = {"persistent": step_p, "kernels": g_k.replay, "fused": step_f}[form]
    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()

    clocks = ClockSampler(local)
    clocks.start()
    local_ms = time_fn(step, args.steps, world)
    clk = clocks.stop()
    assert V.vox_device_status(True) == 0, "device status after the timed steps"
    max_ms, value = aggregate(local_ms, args.steps, step_bytes, world)
    ms_step = max_ms / args.steps

    # the per-projection GEMV kernel (K1) and the split-KV attention kernel (K4) alone
    reps = max(10, min(200, args.steps))
    gg = dm.capture(dm.gemv_chain)
    for _ in range(3):
        gg.replay()
    ms_g = time_fn(gg.replay, reps, world) / reps
    k1_gbs = dm.gemv_chain_bytes() / (ms_g / 1e3) / 1e9
    pos_now = int(dm.pos.item())
    ga = dm.capture(lambda: dm.attn_chain(pos_now))
    for _ in range(3):
        ga.replay()
    ms_a = time_fn(ga.replay, reps, world) / reps
    attn_bytes = dm.kv_bytes(pos_now)
    if form == "persistent":
        roof = {"bound": "hbm", "kernel": "decoder_step_kernel", "achieved": step_bytes / (local_ms / args.steps / 1e3) / 1e9,
                "algorithmic_bytes_per_launch": step_bytes, "avg_launch_us": local_ms / args.steps * 1e3,
                "launches_timed": args.steps, "traffic": STEP_TRAFFIC_BYTES_PER_LAUNCH,
                "note": "one launch is the whole token step, so the dominant kernel is the step"}
    else:
        launches = dm.gemv_chain_launches()
        roof = {"bound": "hbm", "kernel": "q4_gemv_kernel", "achieved": k1_gbs,
                "algorithmic_bytes_per_launch": dm.gemv_chain_bytes() / launches,
                "avg_launch_us": ms_g / launches * 1e3, "launches_timed": reps * launches,
                "traffic": GEMV_TRAFFIC_BYTES_PER_LAUNCH,
                "note": "the step's 105 GEMV launches (69% of its bytes), timed as a graph of the same launches"}
    roof.update({"peak": peak, "unit": "GB/s", "frac": roof["achieved"] / peak, "peak_source": peak_src})

    # end to end through the C ABI: every step copies the token from pinned
    # host memory, runs the step and reads the new token back
    e2e_steps = max(10, min(args.steps, 500))
    tok_h = torch.empty(1, dtype=torch.int32, pin_memory=True)
    out_h = torch.empty(1, dtype=torch.int32, pin_memory=True)
    tok_h[0] = 17
    s = torch.cuda.current_stream()

    def e2e_step():
        dm.token.copy_(tok_h, non_blocking=True)
        if form == "persistent":
            V.vox_decoder_step(dm.dec, s)
        elif form == "fused":
            step_f()
        else:
            g_k.replay()
        out_h.copy_(dm.token, non_blocking=True)
        s.synchronize()
        tok_h[0] = out_h[0]                                   # the host feeds the token back

    e2e_step()
    e2e_local = time_fn(e2e_step, e2e_steps, world)
    _, e2e_value = aggregate(e2e_local, e2e_steps, step_bytes, world)
    assert V.vox_device_status(True) == 0, "device status after the end-to-end steps"

    # the same without a graph: every step calls the C ABI's kernel-sequence
    # step eagerly (its host-side checks and launches included)
    def e2e_eager_step():
        dm.token.copy_(tok_h, non_blocking=True)
        V.vox_decoder_step_kernels(dm.dec, s)
        out_h.copy_(dm.token, non_blocking=True)
        s.synchronize()
        tok_h[0] = out_h[0]

    e2e_eager_step()
    eager_steps = max(5, min(e2e_steps, 100))
    e2e_eager_local = time_fn(e2e_eager_step, eager_steps, world)
    _, e2e_eager_value = aggregate(e2e_eager_local, eager_steps, step_bytes, world)
    assert V.vox_device_status(True) == 0, "device status after the eager end-to-end steps"

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(args.cpu_seconds)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "q4_0 weights, fp16/bf16 tensor-core inputs, f32 accumulate",
            "data": "synthetic",
            "config": decoder_config(shape, world),
            "launch": {"persistent": "one persistent cooperative launch per step",
                       "fused": f"{dm.step_fused_launches()} launches per step (attention + persistent projection "
                                "segments)",
                       "kernels": f"the {dm.step_kernels_launches()}-launch kernel sequence per step"}[form] +
                      ", replayed from a CUDA graph",
            "roofline": roof,
            "step_form": form,
            "forms_ms_per_step": forms,
            "decoder_ms_per_step": ms_step,
            "hbm_frac_step": value / world / peak,
            "k1_gemv": {"kernel": "q4_gemv_kernel", "launches": dm.gemv_chain_launches(),
                        "us_per_launch": ms_g / dm.gemv_chain_launches() * 1e3, "gbs": k1_gbs,
                        "frac": k1_gbs / peak},
            "k4_attention": {"kernel": "gqa_decode_attn_kernel+attn_combine_kernel", "gbs":
                             attn_bytes / (ms_a / 1e3) / 1e9, "us_per_layer": ms_a / dm.L * 1e3},
            "gpu_launches": {"persistent": dm.step_launches(), "fused": dm.step_fused_launches(),
                             "kernels": dm.step_kernels_launches()}[form] * args.steps,
            "clocks": clk,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": 4, "d2h_bytes_per_step": 4,
                    "ms_per_step": e2e_local / e2e_steps,
                    "api": {"persistent": "vox_decoder_step through the C ABI",
                            "fused": "vox_decoder_step_fused captured once in a CUDA graph, replayed",
                            "kernels": "vox_decoder_step_kernels captured once in a CUDA graph, replayed"}[form] +
                           " each step, token H2D before and D2H after, host synchronised every step"},
            "e2e_eager": {"value": e2e_eager_value, "unit": UNIT, "h2d_bytes_per_step": 4, "d2h_bytes_per_step": 4,
                          "ms_per_step": e2e_eager_local / eager_steps,
                          "api": "vox_decoder_step_kernels called through the C ABI every step (no graph), token "
                                 "H2D before and D2H after, host synchronised every step"},
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    del g_p, g_k, gg, ga
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()
    return 0


def decoder_bytes(shape, filled=FILLED):
    """Algorithmic bytes of one decoder step, from the shapes alone: packed
    Q4_0 weights of every layer and the LM head, one embedding row, and the
    bf16 K and V rows the attention reads after position `filled` is written."""
    D, QD, KVD, F, V = shape.dim, shape.q_dim, shape.kv_dim, shape.ffn, shape.vocab
    per_layer = (QD + 2 * KVD) * D + D * QD + 2 * F * D + D * F
    weights = (shape.n_layers * per_layer + V * D + D) * 18 // 32
    kv = shape.n_layers * 2 * shape.n_kv_heads * min(filled + 1, shape.window) * shape.head_dim * 2
    return weights, kv


def decoder_config(shape, world):
    weights, kv = decoder_bytes(shape)
    return {"workload": "decoder_step_q4_26L_kv8192wrapped_M1", "layers": shape.n_layers,
            "dim": shape.dim, "heads": "32q/8kv x 128", "ffn": shape.ffn, "vocab": shape.vocab,
            "kv_window": shape.window, "kv_filled": FILLED, "bytes_per_step": weights + kv,
            "weight_bytes_per_step": weights, "kv_bytes_per_step": kv,
            "l2": "inputs larger than L2 (2.8 GB per step, no flush)", "replicas": world}


# ------------------------------------------------ supplementary workloads
def graph_of(fn):
    """Capture fn (launches on the current stream) into a CUDA graph after
    one warm-up call on a side stream."""
    import torch

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


def run_encoder(args):
    """The 32-layer encoder chunk (M = 256 rows, dim 1280, 32 heads x 40,
    window 750) plus the 5120 -> 3072 adapter GEMM at 64 rows, and the same
    chunk's Q4_0 GEMMs alone (K2, tcgen05)."""
    import torch

    import synth
    from bit_quantized_transformer_b200 import build

    build.build()
    from bit_quantized_transformer_b200 import vox as V
    from bit_quantized_transformer_b200 import workloads as WL

    shape = synth.EncoderShape()
    em = WL.EncoderModel(shape, seed=0)
    steps = max(3, min(args.steps, 50))

    def chunk():
        em.reset()
        em.run()

    g = graph_of(chunk)
    for _ in range(max(3, args.warmup)):
        g.replay()
    ms = time_replays(g, steps, 1) / steps

    # the chunk's GEMMs alone: every layer's QKV, O, up, down at M = 256 and the adapter at M = 64
    R, D, F = shape.rows, shape.dim, shape.ffn
    xb = torch.randn(R, F, device="cuda").to(torch.bfloat16)
    yb = torch.empty(R, max(3 * D, F, shape.adapter_out), dtype=torch.bfloat16, device="cuda")
    calls = []
    for l in range(em.L):
        calls += [(em.wqkv[l], R, D, 3 * D), (em.wo[l], R, D, D), (em.wup[l], R, D, F), (em.wdown[l], R, F, D)]
    calls.append((em.adapter, R // shape.downsample, shape.downsample * D, shape.adapter_out))
    calls.append((em.adapter2, R // shape.downsample, shape.adapter_out, shape.adapter_out))

    def gemms():
        for w, m, k, n in calls:
            V.vox_q4_gemm(w, xb, V.VOX_BF16, m, k, yb, V.VOX_BF16, yb.shape[1])

    gg = graph_of(gemms)
    for _ in range(3):
        gg.replay()
    ms_g = time_replays(gg, steps, 1) / steps
    flops = em.gemm_flops()
    peak = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json"))) if os.path.exists(
        os.path.join(ROOT, "MEASURED_PEAKS.json")) else {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
    tf_g = flops / (ms_g / 1e3) / 1e12
    cpu = None
    if not args.no_cpu_baseline:
        import numpy as np

        from oracle import ref

        w0 = synth.encoder_layer_weights(shape, 0, 0)
        mats = [ref.q4_weights(*w0[k]) for k in ("wqkv", "wo", "wup", "wdown")]
        xs = [np.asarray(synth.activations(R, m.shape[1], 0, 90 + i), np.float64) for i, m in enumerate(mats)]
        t0 = time.perf_counter()
        fl = 0
        while time.perf_counter() - t0 < min(args.cpu_seconds, 10.0):
            for x_, m_ in zip(xs, mats):
                x_ @ m_.T
                fl += 2 * x_.shape[0] * m_.shape[0] * m_.shape[1]
        dt = time.perf_counter() - t0
        cpu = {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": omp_threads(), "kind": "oracle",
               "sample": f"encoder layer 0's four GEMMs at M = {R} (fp64 numpy matmul on the exactly dequantised "
                         f"weights, the oracle's route), {fl / 1e9:.0f} GFLOP in {dt:.1f} s"}
    line = {"metric": "encoder chunk Q4_0 GEMM TFLOP/s (bf16 tensor cores)", "value": tf_g, "unit": "TFLOP/s",
            "n_gpus": 1, "steps": steps, "warmup": max(3, args.warmup), "ms_per_step": ms_g,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16 MMA, f32 accumulate",
            "data": "synthetic",
            "config": {"workload": "encoder_chunk_32L_M256_dim1280_plus_adapter_M64", "gemm_flops": flops,
                       "l2": "weights 353.9 MB > L2"},
            "roofline": {"bound": "tensor", "achieved": tf_g, "peak": peak["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": tf_g / peak["bf16_tflops"], "frac_of_sustained": tf_g / peak["bf16_tflops_sustained"],
                         "traffic": None},
            "chunk_ms": ms, "chunk_tflops_gemm_only_numerator": flops / (ms / 1e3) / 1e12,
            "gpu_launches": len(calls) * steps, "cpu_baseline": cpu}
    print(json.dumps(line), flush=True)
    return 0


def run_sweep(args):
    """The decoder projection shapes at M in {1,4,16,64,256} (K1 for
    M <= 8, K2 for M >= 16, and K1 as two M = 8 launches at M = 16 for the
    crossover), over weight copies totalling > 2x L2; then the decode
    attention at KV 512, 4096 and 8192 (wrapped)."""
    import math

    import numpy as np
    import torch

    import synth
    from bit_quantized_transformer_b200 import build

    build.build()
    from bit_quantized_transformer_b200 import vox as V
    from bit_quantized_transformer_b200 import workloads as WL

    shapes = [(6144, 3072), (3072, 4096), (18432, 3072), (3072, 9216), (131072, 3072)]
    Ms = [1, 4, 16, 64, 256]
    reps = 3
    out = {}
    cross = {}
    x32 = torch.randn(256, 9216, device="cuda")
    xbf = x32.to(torch.bfloat16)
    y = torch.empty(256 * 131072, device="cuda")
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    for n, k in shapes:
        qs, d = synth.q4_blocks(n, k, 0, 77)
        packed, w0 = WL.pack_q4(qs, d, "cuda")
        nbytes = packed.numel()
        copies = max(2, int(math.ceil(300e6 / nbytes)))
        keep = [packed] + [packed.clone() for _ in range(copies - 1)]
        wts = [V.weight(t, n, k) for t in keep]
        res = {}
        for M in Ms + ["16_gemv"] + [f"matmul_{mm}" for mm in Ms]:
            if isinstance(M, str) and M.startswith("matmul_"):
                mm = int(M.split("_")[1])
                wsm = torch.zeros(V.vox_q4_matmul_workspace(wts[0], mm, None), dtype=torch.uint8, device="cuda")

                def fn(mm=mm, wsm=wsm):
                    for w in wts:
                        V.vox_q4_matmul(w, x32, mm, 9216, y, n, None, wsm, wsm.numel())
            elif M == "16_gemv":
                def fn():
                    for w in wts:
                        for h in range(2):
                            V.vox_q4_gemv(w, x32[8 * h:], 8, 9216, y, n, None, ws, 4096)
            elif M <= 8:
                def fn(M=M):
                    for w in wts:
                        V.vox_q4_gemv(w, x32, M, 9216, y, n, None, ws, 4096)
            else:
                def fn(M=M):
                    for w in wts:
                        V.vox_q4_gemm(w, xbf, V.VOX_BF16, M, 9216, y, V.VOX_F32, n)
            g = graph_of(fn)
            g.replay()
            us = time_replays(g, reps, 1) / (reps * copies) * 1e3
            m = 16 if M == "16_gemv" else (int(M.split("_")[1]) if isinstance(M, str) else M)
            res[str(M)] = {"us": us, "weight_gbs": nbytes / us / 1e3, "tflops": 2 * m * n * k / us / 1e6}
            del g
        out[f"{n}x{k}"] = res
        cross[f"{n}x{k}"] = "K2 (tcgen05 GEMM) faster at M=16" if res["16"]["us"] < res["16_gemv"]["us"] else \
            "K1 (two M=8 GEMVs) faster at M=16"
        del keep, wts
        torch.cuda.empty_cache()
    # attention at three cache lengths
    n_q, n_kv, hd, W = 32, 8, 128, 8192
    NL = 26
    caches = [(torch.randn(n_kv, W, hd, device="cuda").to(torch.bfloat16),
               torch.randn(n_kv, W, hd, device="cuda").to(torch.bfloat16)) for _ in range(NL)]
    q = torch.randn(n_q, hd, device="cuda")
    o = torch.empty(n_q, hd, device="cuda")
    wsb = V.vox_gqa_decode_attn_workspace(n_q, n_kv, hd, W)
    wsa = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    attn = {}
    for pos in (511, 4095, W + 300):
        def fa(pos=pos):
            for l in range(NL):
                V.vox_gqa_decode_attn(q, caches[l][0], caches[l][1], o, n_q, n_kv, hd, W, pos, 1 / math.sqrt(hd),
                                      wsa, wsb)
        g = graph_of(fa)
        g.replay()
        us = time_replays(g, 5, 1) / (5 * NL) * 1e3
        nb = 2 * n_kv * min(pos + 1, W) * hd * 2
        attn[str(min(pos + 1, W)) + (" wrapped" if pos >= W else "")] = {"us_per_layer": us, "gbs": nb / us / 1e3}
        del g
    assert V.vox_device_status(True) == 0
    peak, peak_src = measured_peaks()
    lm1 = out["131072x3072"]["1"]["weight_gbs"]
    line = {"metric": "decoder-shape sweep: weight GB/s and TFLOP/s per M; attention GB/s per KV length",
            "value": out["131072x3072"]["1"]["weight_gbs"], "unit": "GB/s", "n_gpus": 1, "steps": reps,
            "warmup": 1, "ms_per_step": None, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "q4_0 weights; fp16 (K1) / bf16 (K2) tensor-core inputs; f32 accumulate", "data": "synthetic",
            "config": {"workload": "decoder_shapes_M_sweep_and_attention_kv_sweep", "M": Ms,
                       "l2": "weight copies > 2x L2 per shape"},
            "sweep": out, "crossover": cross, "attention": attn,
            "roofline": {"bound": "hbm", "kernel": "q4_gemv_kernel (LM head, M = 1)", "achieved": lm1, "peak": peak,
                         "unit": "GB/s", "frac": lm1 / peak, "traffic": None, "peak_source": peak_src},
            "dispatch": "vox_q4_matmul: the GEMV for M <= 8, the tcgen05 GEMM above (entries matmul_M)"}
    print(json.dumps(line), flush=True)
    return 0


def run_gemv(args):
    """Config 0: the single Q4_0 GEMV, 4096 x 3072 at M = 1 (weights seed 0,
    activation N(0, 1)), through vox_q4_gemv.  Timed two ways: a CUDA graph of
    launches cycling over distinct weight copies that total more than 2x L2
    (every launch streams weights that are not in L2), and single calls, each
    after an L2 flush (a 256 MB write) between its CUDA events."""
    import numpy as np
    import torch

    import synth
    from bit_quantized_transformer_b200 import build

    build.build()
    from bit_quantized_transformer_b200 import vox as V
    from bit_quantized_transformer_b200 import workloads as WL
    from oracle import ref

    n, k = 4096, 3072
    qs, d = synth.q4_blocks(n, k, 0, synth.X_ID + 100)
    xh = synth.activations(1, k, 0, synth.X_ID)
    packed, w0 = WL.pack_q4(qs, d, "cuda")
    nbytes = packed.numel()
    copies = 40                                           # 40 x 7.08 MB = 283 MB > 2 x 126 MB
    keep = [packed] + [packed.clone() for _ in range(copies - 1)]
    ws_ = [V.weight(t, n, k) for t in keep]
    x = WL.to_dev(xh, "cuda")
    y = torch.empty(1, n, device="cuda")
    wsb = V.vox_q4_gemv_workspace(w0, 1, None)
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    V.vox_q4_gemv(w0, x, 1, k, y, n, None, ws, wsb)
    torch.cuda.synchronize()
    W = ref.q4_weights(qs, d)
    err = ref.gemv_error(y.cpu().numpy(), xh.astype(np.float64) @ W.T, xh, W)
    assert err <= 2e-3, err

    def chain():
        for w in ws_:
            V.vox_q4_gemv(w, x, 1, k, y, n, None, ws, wsb)

    g = graph_of(chain)
    for _ in range(max(3, args.warmup)):
        g.replay()
    reps = max(3, args.steps)
    clocks = ClockSampler(0)
    clocks.start()
    ms = time_fn(g.replay, reps, 1)
    clk = clocks.stop()
    us = ms / (reps * copies) * 1e3
    gbs = nbytes / us / 1e3
    # cold single calls: flush L2 with a 256 MB write, then time one launch
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device="cuda")
    s = torch.cuda.current_stream()
    cold = []
    for i in range(max(5, min(args.steps, 50))):
        flush.fill_(float(i))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        V.vox_q4_gemv(ws_[i % copies], x, 1, k, y, n, None, ws, wsb)
        e1.record(s)
        torch.cuda.synchronize()
        cold.append(e0.elapsed_time(e1) * 1e3)
    cold_us = statistics.median(cold)
    peak, peak_src = measured_peaks()
    cpu = None
    if not args.no_cpu_baseline:
        t0 = time.perf_counter()
        done = 0
        while time.perf_counter() - t0 < min(args.cpu_seconds, 10.0):
            ref.c_matvec(qs, d, xh)
            done += 1
        dt = time.perf_counter() - t0
        cpu = {"value": done * nbytes / dt / 1e9, "unit": "GB/s", "cores": omp_threads(), "kind": "oracle",
               "sample": f"{done} full 4096 x 3072 GEMVs (fp64 C oracle, OpenMP over rows) in {dt:.1f} s"}
    line = {"metric": "Q4_0 GEMV weight GB/s, 4096 x 3072, M = 1", "value": gbs, "unit": "GB/s", "n_gpus": 1,
            "steps": reps, "warmup": max(3, args.warmup), "ms_per_step": ms / reps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "q4_0 weights, fp16 tensor-core inputs, f32 accumulate",
            "data": "synthetic",
            "config": {"workload": "q4_gemv_4096x3072_M1", "weight_bytes": nbytes, "copies": copies,
                       "l2": "graph of launches over 40 weight copies (283 MB > 2x L2); cold calls after a 256 MB "
                             "L2 flush"},
            "roofline": {"bound": "hbm", "kernel": "q4_gemv_kernel", "achieved": gbs, "peak": peak, "unit": "GB/s",
                         "frac": gbs / peak, "traffic": None, "peak_source": peak_src,
                         "avg_launch_us": us, "ideal_us": nbytes / peak / 1e3},
            "cold_call": {"us": cold_us, "gbs": nbytes / cold_us / 1e3, "calls": len(cold)},
            "parity_error": err, "gpu_launches": reps * copies, "clocks": clk, "cpu_baseline": cpu}
    print(json.dumps(line), flush=True)
    return 0


def run_layer(args):
    """Config 1: one decoder layer at M = 1, KV length 1024 (each step writes
    one more position and attends over 1025 keys), all Q4_0 weights drawn as in
    config 0.  Four distinct layers (rotated, 279 MB > 2x L2) run as one decoder
    step whose embedding table and LM head have 16 rows (27 KB, under 0.1% of
    the step); the per-layer time is the step time / 4, in the faster of the
    step's two forms.  The window is 1025 positions, already wrapped, so every
    step attends over exactly 1025 keys."""
    import torch

    import synth
    from bit_quantized_transformer_b200 import build

    build.build()
    from bit_quantized_transformer_b200 import vox as V
    from bit_quantized_transformer_b200 import workloads as WL

    shape = synth.DecoderShape(n_layers=4, vocab=16, window=1025)
    dm = WL.DecoderModel(shape, seed=0, filled=2 * 1025, token=3)
    wbytes, kv = decoder_bytes(shape, 2 * 1025)
    layer_bytes = (wbytes - (shape.vocab * shape.dim + shape.dim) * 18 // 32 + kv) // shape.n_layers
    step_bytes = wbytes + kv
    g = try_graph(dm.step)
    step_p = g.replay if g is not None else dm.step
    gk = dm.capture(dm.step_kernels)
    forms = {}
    for name, fn in (("persistent", step_p), ("kernels", gk.replay)):
        for _ in range(max(3, args.warmup)):
            fn()
        torch.cuda.synchronize()
        assert V.vox_device_status(True) == 0
        forms[name] = time_fn(fn, 10, 1) / 10 / shape.n_layers * 1e3
    form = min(forms, key=forms.get)
    step = step_p if form == "persistent" else gk.replay
    reps = max(3, args.steps)
    clocks = ClockSampler(0)
    clocks.start()
    ms = time_fn(step, reps, 1)
    clk = clocks.stop()
    assert V.vox_device_status(True) == 0
    us_layer = ms / reps / shape.n_layers * 1e3
    gbs = layer_bytes / us_layer / 1e3
    peak, peak_src = measured_peaks()
    cpu = None
    if not args.no_cpu_baseline:
        b, t, n_done, threads = oracle_decoder_sample(min(args.cpu_seconds, 15.0), layers=4, filled=1024)
        cpu = {"value": b / t / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
               "sample": f"{n_done} decoder-layer passes at KV 1025 (fp64 C oracle), {b / 1e6:.1f} MB in {t:.1f} s"}
    line = {"metric": "decoder layer GB/s (weights + KV), M = 1, KV 1024", "value": gbs, "unit": "GB/s",
            "n_gpus": 1, "steps": reps, "warmup": max(3, args.warmup), "ms_per_step": ms / reps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "q4_0 weights, fp16/bf16 tensor-core inputs, f32 accumulate", "data": "synthetic",
            "config": {"workload": "decoder_layer_q4_kv1024_M1", "layers_rotated": shape.n_layers,
                       "bytes_per_layer": layer_bytes, "kv_keys": 1025,
                       "l2": "4 distinct layers per step (279 MB > 2x L2), no flush"},
            "us_per_layer": us_layer,
            "roofline": {"bound": "hbm", "kernel": "decoder_step_kernel" if form == "persistent" else
                         "the layer's kernel sequence", "achieved": gbs, "peak": peak,
                         "unit": "GB/s", "frac": gbs / peak, "traffic": None, "peak_source": peak_src},
            "step_form": form, "forms_us_per_layer": forms,
            "gpu_launches": reps * (dm.step_launches() if form == "persistent" else dm.step_kernels_launches()),
            "clocks": clk, "cpu_baseline": cpu}
    print(json.dumps(line), flush=True)
    return 0


def run_batch(args):
    """Batched decode: --seqs sequences, each with its own 8192-slot rolling
    cache in 64-slot pages (filled past one wrap, positions 8192 + 300 + 37 s),
    stepped together through the 26-layer decoder: every weight is streamed
    once per step for all sequences (the GEMV at m = seqs rows), the
    attention reads every sequence's cache.  One step = one replay of the
    captured vox_decoder_batch_step graph.  Reports tokens/s and the step's
    algorithmic GB/s (weights once + every sequence's cache)."""
    import torch

    import synth
    from bit_quantized_transformer_b200 import build

    build.build()
    from bit_quantized_transformer_b200 import vox as V
    from bit_quantized_transformer_b200 import workloads as WL

    n = max(1, min(8, args.seqs))
    shape = synth.DecoderShape()
    positions = [FILLED + 37 * s for s in range(n)]
    tokens = [(17 + 7919 * s) % shape.vocab for s in range(n)]
    bm = WL.BatchDecoderModel(shape, n, positions, tokens, device_fill=True)
    step_bytes = bm.weight_bytes() + bm.kv_bytes(positions)
    g = bm.capture()
    for _ in range(max(3, args.warmup)):
        g.replay()
    torch.cuda.synchronize()
    assert V.vox_device_status(True) == 0
    reps = max(3, args.steps)
    clocks = ClockSampler(0)
    clocks.start()
    ms = time_fn(g.replay, reps, 1)
    clk = clocks.stop()
    assert V.vox_device_status(True) == 0
    ms_step = ms / reps
    gbs = step_bytes / (ms_step / 1e3) / 1e9
    peak, peak_src = measured_peaks()
    # end to end through the API: tokens in from pinned host memory, next tokens out, every step
    tok_h = torch.tensor(tokens, dtype=torch.int32).pin_memory()
    out_h = torch.empty(n, dtype=torch.int32).pin_memory()

    def e2e_step():
        bm.token.copy_(tok_h, non_blocking=True)
        g.replay()
        out_h.copy_(bm.token, non_blocking=True)
        torch.cuda.current_stream().synchronize()

    e2e_n = max(3, min(reps, 50))
    t0 = time.perf_counter()
    for _ in range(e2e_n):
        e2e_step()
    e2e_ms = (time.perf_counter() - t0) * 1e3 / e2e_n
    assert V.vox_device_status(True) == 0
    del g
    line = {"metric": "batched decode tokens/s (sequences x steps / s), paged per-sequence caches",
            "value": n * 1e3 / ms_step, "unit": "tokens/s", "n_gpus": 1, "steps": reps,
            "warmup": max(3, args.warmup), "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "q4_0 weights, fp16/bf16 tensor-core inputs, f32 accumulate",
            "data": "synthetic (pools drawn on the device)",
            "config": {"workload": f"decoder_batch_q4_26L_kv8192wrapped_{n}seq_paged", "sequences": n,
                       "positions": positions, "page_slots": 64, "pages": bm.n_pages,
                       "bytes_per_step": step_bytes, "l2": "inputs larger than L2 (no flush)"},
            "gbs": gbs, "hbm_frac": gbs / peak,
            "roofline": {"bound": "hbm", "kernel": "the batched step's kernel sequence", "achieved": gbs,
                         "peak": peak, "unit": "GB/s", "frac": gbs / peak, "traffic": None,
                         "peak_source": peak_src},
            "gpu_launches": reps * bm.launches(), "clocks": clk,
            "e2e": {"value": n * 1e3 / e2e_ms, "unit": "tokens/s", "h2d_bytes_per_step": 4 * n,
                    "d2h_bytes_per_step": 4 * n, "ms_per_step": e2e_ms,
                    "api": "vox_decoder_batch_step graph replay, tokens H2D before and D2H after every step"}}
    print(json.dumps(line), flush=True)
    return 0


def omp_threads():
    return int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))


def run_kernel_case(args):
    """A few launches of one kernel on one case that holds well under 1 GB on
    the device (seeded synthetic inputs as in the decoder workload), for an
    ncu capture; checks the device status word and prints one JSON line.
      gemv N K   : the Q4_0 GEMV, M = 1, no epilogue, on one packed N x K weight
      attn POS   : split-KV decode attention, 32 query / 8 kv heads x 128,
                   8192-slot bf16 rolling cache, after position POS was written
      gemm N K M : the Q4_0 GEMM (tcgen05), M bf16 activation rows, bf16 output"""
    import math

    import torch

    import synth
    from bit_quantized_transformer_b200 import build

    build.build()
    from bit_quantized_transformer_b200 import vox as V
    from bit_quantized_transformer_b200 import workloads as WL

    shp = args.shape or {"gemv": [4096, 3072], "attn": [8492], "gemm": [131072, 3072, 256], "step": [2],
                         "stepk": [26], "encoder": [32]}[args.kernel]
    if args.kernel == "stepk":
        shape = synth.DecoderShape(n_layers=shp[0])
        dm = WL.DecoderModel(shape, seed=0, filled=FILLED, token=17)
        for _ in range(args.launches):
            dm.step_kernels()
        what = {"kernel": "decoder step kernel sequence", "layers": shp[0],
                "launches_per_step": dm.step_kernels_launches(),
                "bytes_per_step": dm.weight_bytes() + dm.kv_bytes(FILLED)}
    elif args.kernel == "encoder":
        shape = synth.EncoderShape(n_layers=shp[0])
        em = WL.EncoderModel(shape, seed=0)
        for _ in range(args.launches):
            em.reset()
            em.run()
        what = {"kernel": "encoder chunk", "layers": shp[0], "gemm_flop_per_chunk": em.gemm_flops()}
    elif args.kernel == "step":
        shape = synth.DecoderShape(n_layers=shp[0])
        dm = WL.DecoderModel(shape, seed=0, filled=FILLED, token=17)
        for _ in range(args.launches):
            dm.step()
        what = {"kernel": "decoder_step_kernel", "layers": shp[0],
                "bytes_per_launch": dm.weight_bytes() + dm.kv_bytes(FILLED)}
    elif args.kernel == "gemv":
        n, k = shp[0], shp[1]
        qs, d = synth.q4_blocks(n, k, 0, 77)
        packed, w = WL.pack_q4(qs, d, "cuda")
        x = WL.to_dev(synth.activations(1, k, 0, 78), "cuda")
        y = torch.empty(1, n, device="cuda")
        wsb = V.vox_q4_gemv_workspace(w, 1, None)
        ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
        for _ in range(args.launches):
            V.vox_q4_gemv(w, x, 1, k, y, n, None, ws, wsb)
        what = {"kernel": "q4_gemv_kernel", "n": n, "k": k, "weight_bytes_per_launch": packed.numel()}
    elif args.kernel == "gemm":
        n, k, m = shp[0], shp[1], shp[2]
        qs, d = synth.q4_blocks(n, k, 0, 79)
        packed, w = WL.pack_q4(qs, d, "cuda")
        x = WL.bf16_dev(synth.bf16_normal((m, k), 0, 80), "cuda")
        y = torch.empty(m, n, dtype=torch.bfloat16, device="cuda")
        for _ in range(args.launches):
            V.vox_q4_gemm(w, x, V.VOX_BF16, m, k, y, V.VOX_BF16, n)
        what = {"kernel": "q4_gemm_kernel", "n": n, "k": k, "m": m, "flop_per_launch": 2 * m * n * k}
    else:
        pos = shp[0]
        n_q, n_kv, hd, W = 32, 8, 128, 8192
        kc = torch.randn(n_kv, W, hd, device="cuda").to(torch.bfloat16)
        vc = torch.randn(n_kv, W, hd, device="cuda").to(torch.bfloat16)
        q = torch.randn(n_q, hd, device="cuda")
        out = torch.empty(n_q, hd, device="cuda")
        wsb = V.vox_gqa_decode_attn_workspace(n_q, n_kv, hd, W)
        ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
        for _ in range(args.launches):
            V.vox_gqa_decode_attn(q, kc, vc, out, n_q, n_kv, hd, W, pos, 1.0 / math.sqrt(hd), ws, wsb)
        what = {"kernel": "gqa_decode_attn_kernel", "pos": pos,
                "cache_bytes_per_launch": 2 * n_kv * min(pos + 1, W) * hd * 2}
    torch.cuda.synchronize()
    assert V.vox_device_status(True) == 0
    print(json.dumps({"workload": "kernel case", "launches": args.launches, **what}), flush=True)
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    if args.workload == "encoder":
        return run_encoder(args)
    if args.workload == "sweep":
        return run_sweep(args)
    if args.workload == "kernel":
        return run_kernel_case(args)
    if args.workload == "gemv":
        return run_gemv(args)
    if args.workload == "layer":
        return run_layer(args)
    if args.workload == "batch":
        return run_batch(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
