#!/usr/bin/env python
"""Throughput of the Ecco block codec on one or more B200s (one process per GPU).

Default workload (`--workload longctx`, the largest configuration): a
32-layer long-context KV cache, K and V of every layer [1, 8, 131072, 128]
bf16 (17.2 GB).  A step appends one token to every layer's K and V (512
groups, encoded into the compressed cache) and decodes the whole compressed
cache back to bf16 (67,108,864 blocks); each direction is one multi-segment
call (`encode_multi`, `decode_multi`: 64 tensors in one launch).  Other
workloads: `kv` (one Llama-3-8B-shaped layer, K and V [8, 8, 4096, 128]:
encode of the last 64 tokens + decode of the whole cache), `c1` (256 x 1024
matrix, encode + decode), `mlp` (14336 x 4096 weight: encode, decode, fused
decode+GEMV at batch 1 and 16), `model` (32 layers x 7 weights, encode and
decode of the whole set),
`attn` (one-token append + staged decode+attention over the compressed cache of
the `kv` layer, 32 query heads), `select` (encode of the `kv` layer with
full-MSE pattern selection, plus a quality study of min/max vs full-MSE
selection with 64 and 16 patterns), `act` (the 2x activation format: [8192,
4096] hidden states in 64-value groups, encode + decode).

Prints ONE JSON line (rank 0).  `value` is whole-job bf16 GB/s: bf16 bytes the
step decodes plus bf16 bytes it encodes, over all ranks, per second of device
time (CUDA events on the launching stream, max over ranks).  L2 is flushed
between timed steps by writing a 256 MiB buffer outside the step's events.
`--impl reference` times the CPU oracle on a bounded sample of the same step.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decoded GB/s (bf16 out) & encode GB/s, % of HBM roofline, bit-exact vs oracle"
TABLE_BLOB_BYTES = 7952  # one tensor's stored tables: S_t, 64 x 15 centroids, 64 x 4 x 16 code lengths
FALLBACK_HBM_GBS = 6650.0


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ecco", choices=["ecco", "reference"])
    ap.add_argument("--workload", default="longctx", choices=["kv", "c1", "mlp", "model", "longctx", "attn", "select", "act"])
    ap.add_argument("--attention", default="staged", choices=["staged", "fused"],
                    help="attn workload: decode_attention_staged (default) or the single fused kernel")
    ap.add_argument("--decoder", default="serial", choices=["serial", "speculative"],
                    help="kv workload: decode with the thread-per-block walk (default) or the warp-parallel "
                         "speculative decoder (ecco_decode_speculative, one launch per tensor)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target oracle time for cpu_baseline")
    ap.add_argument("--layers", type=int, default=32,
                    help="model / longctx: layers built (32 = the full configuration; fewer for profiling captures)")
    return ap.parse_args()


def peaks():
    """HBM copy bandwidth (GB/s) from MEASURED_PEAKS.json's hbm_gbs (a number,
    or an object holding one under value / gbs / burst), else the fallback."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if not os.path.exists(p):
        return FALLBACK_HBM_GBS, "fallback"
    try:
        with open(p) as f:
            v = json.load(f)["hbm_gbs"]
        if isinstance(v, dict):
            v = next(v[k] for k in ("value", "gbs", "burst") if k in v)
        v = float(v)
        if v > 0:
            return v, "measured"
    except (OSError, ValueError, KeyError, TypeError, StopIteration):
        pass
    return FALLBACK_HBM_GBS, "fallback (MEASURED_PEAKS.json has no usable hbm_gbs)"


# ------------------------------------------------------------------ clocks
class Clocks:
    """Polls NVML (read-only) every millisecond while the timed region runs:
    SM clock, its maximum, and the active clock-event (throttle) reasons."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap"}

    def __init__(self, torch_dev):
        self.dev = torch_dev
        self.samples = []
        self.reasons = set()
        self.h = None
        self._stop = None
        self._th = None

    def _handle(self):
        import pynvml
        pynvml.nvmlInit()
        try:
            import torch
            p = torch.cuda.get_device_properties(self.dev)
            bus = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
            return pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return pynvml.nvmlDeviceGetHandleByIndex(self.dev.index or 0)

    def start(self):
        import threading
        try:
            import pynvml
            self.h = self._handle()
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # NVML missing: report it, do not guess
            self.h = None
            self.err = str(e)
            return
        self._stop = threading.Event()

        def poll():
            import pynvml
            while not self._stop.is_set():
                try:
                    self.samples.append(pynvml.nvmlDeviceGetClockInfo(self.h, pynvml.NVML_CLOCK_SM))
                    r = pynvml.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                    for bit, name in self.REASONS.items():
                        if r & bit:
                            self.reasons.add(name)
                except Exception:
                    pass
                self._stop.wait(0.001)

        self._th = threading.Thread(target=poll, daemon=True)
        self._th.start()

    def stop(self) -> dict:
        if self.h is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [f"nvml unavailable: {getattr(self, 'err', '')}"]}
        self._stop.set()
        self._th.join(timeout=2)
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ------------------------------------------------------------------ workloads
class Workload:
    name = ""
    desc = ""
    launches_per_step = 0
    stats = None       # ecco_stats counters of one encode of the whole workload (setup, untimed)
    n_tensors = 1      # tensors with their own table blob
    group = 128        # values per group

    def stats_summary(self):
        """Clipping, padding and compression of the workload's blocks: the
        review page's Fig. 10 (padding and clipping ratios) and "Core claim"
        (memory reduction) quantities, from the encoder's own counters."""
        if not self.stats:
            return None
        st = self.stats
        n = max(1, st["n_groups"])
        raw = st["n_groups"] * self.group * 2
        blocks = st["n_groups"] * 64
        tables = self.n_tensors * TABLE_BLOB_BYTES
        return {"groups": st["n_groups"], "clip_ratio": round(st["n_clipped"] / n, 5),
                "pad_ratio": round(st["n_padded"] / n, 5), "records_per_block": round(st["n_records"] / n, 4),
                "payload_bits_per_block": round(st["payload_bits"] / n, 2),
                "zero_blocks": st["n_zero"], "nonfinite_values": st["n_nonfinite"],
                "compression_ratio": round(raw / blocks, 4),
                "compression_ratio_with_tables": round(raw / (blocks + tables), 4),
                "table_blob_bytes": TABLE_BLOB_BYTES, "tensors": self.n_tensors}

    def bytes_decoded(self) -> int:      # bf16 bytes written by decode per step
        return 0

    def cpu_frac(self) -> float:         # fraction of a step the oracle samples (~1 s of host work)
        return 1.0

    def bytes_encoded(self) -> int:      # bf16 bytes read by encode per step
        return 0


class LayerStream:
    """End-to-end leg of the two large workloads, streamed layer by layer.

    Per layer: host-to-device copies of that layer's inputs (from pinned host
    memory) on one stream, the library calls on the current stream once those
    copies landed, device-to-host copies of that layer's results on a third
    stream once the calls finished.  Copies of one layer overlap the calls of
    the next.  Inputs come from pinned host copies of the whole step's inputs;
    results go to two pinned staging buffers used by alternate layers (the host
    does not read them while the step is timed), so every input byte crosses
    to the device and every result byte crosses back once per step."""

    def __init__(self, torch, dev, layers):
        """layers: [(ins, run, outs)]: ins = [(host pinned, device)] pairs,
        run() enqueues the layer's library calls on the current stream, outs =
        device tensors to copy back."""
        self.torch, self.layers = torch, layers
        self.s_in, self.s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        most = max(sum(t.numel() * t.element_size() for t in outs) for _, _, outs in layers)
        self.stage = [torch.empty(most, dtype=torch.uint8).pin_memory() for _ in range(2)]
        self.h2d = sum(h.numel() * h.element_size() for ins, _, _ in layers for h, _ in ins)
        self.d2h = sum(t.numel() * t.element_size() for _, _, outs in layers for t in outs)

    def step(self):
        torch = self.torch
        main = torch.cuda.current_stream()
        go = torch.cuda.Event()
        go.record(main)
        self.s_in.wait_event(go)
        for li, (ins, run, outs) in enumerate(self.layers):
            with torch.cuda.stream(self.s_in):
                for h, d in ins:
                    d.copy_(h, non_blocking=True)
            landed = torch.cuda.Event()
            landed.record(self.s_in)
            main.wait_event(landed)
            run()
            ran = torch.cuda.Event()
            ran.record(main)
            self.s_out.wait_event(ran)
            with torch.cuda.stream(self.s_out):
                st, off = self.stage[li % 2], 0
                for t in outs:
                    nb = t.numel() * t.element_size()
                    st[off:off + nb].copy_(t.reshape(-1).view(torch.uint8), non_blocking=True)
                    off += nb
        done = torch.cuda.Event()
        done.record(self.s_out)
        main.wait_event(done)


def _events(torch):
    return torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)


class KVWorkload(Workload):
    """One layer of KV cache: encode 64 new tokens, decode the whole cache."""
    name = "kv"
    desc = ("Llama-3-8B-shaped one-layer KV cache, K and V each [8, 8, 4096, 128] bf16: "
            "encode the last 64 tokens (8,192 groups) + decode the full cache (524,288 blocks)")
    B, H, S, D, T = 8, 8, 4096, 128, 64
    speculative = False  # decode through ecco_decode_speculative instead

    def __init__(self, dev, seed_offset=0):
        import torch
        import workloads as W
        import entropy_coded_kv_b200 as ecco
        from entropy_coded_kv_b200.calib import learn_tables
        self.torch, self.ecco, self.dev = torch, ecco, dev
        K, V = W.c2_kv(device=dev, seed=1 + seed_offset)
        Kc, Vc = W.c2_calibration(device=dev, seed=2 + seed_offset)
        self.tables = [ecco.Tables(learn_tables(Kc, seed=0), dev), ecco.Tables(learn_tables(Vc, seed=0), dev)]
        self.rows = self.B * self.H
        self.n = self.rows * self.S
        self.caches = [K, V]
        st = ecco.new_stats(dev)
        self.blocks = [ecco.encode(K, self.tables[0], stats=st), ecco.encode(V, self.tables[1], stats=st)]
        self.stats, self.n_tensors = ecco.read_stats(st), 2
        self.new = [K.view(self.rows, self.S, self.D)[:, self.S - self.T:].contiguous(),
                    V.view(self.rows, self.S, self.D)[:, self.S - self.T:].contiguous()]
        self.out = [torch.empty((self.n, 128), dtype=torch.bfloat16, device=dev) for _ in range(2)]
        self.append = ecco.kv_append_desc(self.rows, self.T, self.S, self.S - self.T)
        self.app = [ecco.Seg(self.tables[i], self.new[i], self.blocks[i], self.append) for i in range(2)]
        self.dec = [ecco.Seg(self.tables[i], self.blocks[i], self.out[i]) for i in range(2)]
        self.launches_per_step = 3 if self.speculative else 2
        if self.speculative:
            self.desc = self.desc + "; decode by the warp-parallel speculative decoder (one launch per tensor)"
        self.dec_ms = []

    def _decode(self):
        if self.speculative:
            for i in range(2):
                self.ecco.decode(self.blocks[i], self.tables[i], out=self.out[i], speculative=True)
        else:
            self.ecco.decode_multi(self.dec)

    def bytes_decoded(self):
        return 2 * self.n * 256

    def bytes_encoded(self):
        return 2 * self.rows * self.T * 256

    def step(self, record=False):
        """K and V appended in one multi-segment launch, both caches decoded in one."""
        e = self.ecco
        e.encode_multi(self.app)
        if record:
            a, b = _events(self.torch)
            a.record()
        self._decode()
        if record:
            b.record()
            self.dec_ms.append((a, b))

    def dominant(self):
        """(kernel name, algorithmic bytes per launch, launch ms list)."""
        self.torch.cuda.synchronize()
        ms = [a.elapsed_time(b) for a, b in self.dec_ms]
        return ("decode_spec_kernel" if self.speculative else "decode_kernel"), 2 * self.n * (64 + 256), ms

    # ---- end to end through the public API with host buffers
    def e2e_setup(self):
        torch = self.torch
        self.h_new = [t.cpu().pin_memory() for t in self.new]
        self.h_blocks = [b.cpu().pin_memory() for b in self.blocks]
        self.h_out = [torch.empty((self.n, 128), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        self.d_new = [torch.empty_like(t) for t in self.new]
        self.e2e_app = [self.ecco.Seg(self.tables[i], self.d_new[i], self.blocks[i], self.append) for i in range(2)]
        self.h2d = sum(t.numel() * t.element_size() for t in self.h_new + self.h_blocks)
        self.d2h = sum(t.numel() * t.element_size() for t in self.h_out)

    def e2e_step(self):
        e = self.ecco
        for i in range(2):
            self.d_new[i].copy_(self.h_new[i], non_blocking=True)
            self.blocks[i].copy_(self.h_blocks[i], non_blocking=True)
        e.encode_multi(self.e2e_app)
        self._decode()
        for i in range(2):
            self.h_out[i].copy_(self.out[i], non_blocking=True)

    # ---- CPU oracle on a bounded sample of the same step
    def cpu_sample(self, frac):
        import numpy as np
        import workloads as W
        n_dec = max(64, int(self.n * frac))
        n_enc = max(8, int(self.rows * self.T * frac))
        xs = [W.bf16_bits(self.new[i].view(-1, 128)[:n_enc]) for i in range(2)]
        bl = [self.blocks[i][:n_dec].cpu().numpy() for i in range(2)]
        blobs = [t.blob for t in self.tables]
        return {"enc": [(blobs[i], xs[i]) for i in range(2)], "dec": [(blobs[i], bl[i]) for i in range(2)],
                "bytes": 2 * n_dec * 256 + 2 * n_enc * 256,
                "what": f"encode {2 * n_enc} groups + decode {2 * n_dec} blocks (1/{round(1 / frac)} of a step)"}


class C1Workload(Workload):
    name = "c1"
    desc = "256 x 1024 bf16 matrix, N(0, 0.02^2) + 0.1% +-20 sigma outliers: encode + decode"

    def __init__(self, dev, seed_offset=0):
        import torch
        import workloads as W
        import entropy_coded_kv_b200 as ecco
        from entropy_coded_kv_b200.calib import learn_tables
        self.torch, self.ecco, self.dev = torch, ecco, dev
        self.x = W.c1_matrix(device=dev, seed=0 + seed_offset)
        self.tables = ecco.Tables(learn_tables(W.c1_matrix(seed=0 + seed_offset)), dev)
        st = ecco.new_stats(dev)
        self.blocks = ecco.encode(self.x, self.tables, stats=st)
        self.stats = ecco.read_stats(st)
        self.out = torch.empty((2048, 128), dtype=torch.bfloat16, device=dev)
        self.launches_per_step = 2
        self.dec_ms = []

    def bytes_decoded(self):
        return 2048 * 256

    def bytes_encoded(self):
        return 2048 * 256

    def step(self, record=False):
        self.ecco.encode(self.x, self.tables, out=self.blocks)
        if record:
            a, b = _events(self.torch)
            a.record()
        self.ecco.decode(self.blocks, self.tables, out=self.out)
        if record:
            b.record()
            self.dec_ms.append((a, b))

    def dominant(self):
        self.torch.cuda.synchronize()
        return "decode_kernel", 2048 * 320, [a.elapsed_time(b) for a, b in self.dec_ms]

    def e2e_setup(self):
        self.hx = self.x.cpu().pin_memory()
        self.hy = self.torch.empty_like(self.out, device="cpu").pin_memory()
        self.dx = self.torch.empty_like(self.x)
        self.h2d, self.d2h = self.hx.numel() * 2, self.hy.numel() * 2

    def e2e_step(self):
        self.dx.copy_(self.hx, non_blocking=True)
        self.ecco.encode(self.dx, self.tables, out=self.blocks)
        self.ecco.decode(self.blocks, self.tables, out=self.out)
        self.hy.copy_(self.out, non_blocking=True)

    def cpu_sample(self, frac):
        import workloads as W
        xb = W.bf16_bits(self.x)
        return {"enc": [(self.tables.blob, xb)], "dec": [(self.tables.blob, self.blocks.cpu().numpy())],
                "bytes": 2 * 2048 * 256, "what": "the whole step (encode 2048 groups + decode 2048 blocks)"}


class MLPWorkload(Workload):
    name = "mlp"
    desc = ("14336 x 4096 bf16 weight, Student-t(5) x 0.02: encode, decode, fused decode+GEMV "
            "at batch 1 and batch 16")

    def __init__(self, dev, seed_offset=0):
        import torch
        import workloads as W
        import entropy_coded_kv_b200 as ecco
        from entropy_coded_kv_b200.calib import learn_tables
        self.torch, self.ecco, self.dev = torch, ecco, dev
        self.w = W.c3_weight(device=dev, seed=3 + seed_offset)
        self.rows, self.cols = self.w.shape
        self.n = self.rows * self.cols // 128
        self.tables = ecco.Tables(learn_tables(self.w, seed=0), dev)
        st = ecco.new_stats(dev)
        self.blocks = ecco.encode(self.w, self.tables, stats=st)
        self.stats = ecco.read_stats(st)
        self.out = torch.empty((self.n, 128), dtype=torch.bfloat16, device=dev)
        self.x1 = W.activations(self.cols, 1, device=dev)
        self.x16 = W.activations(self.cols, 16, device=dev)
        self.y1 = torch.empty((1, self.rows), dtype=torch.float32, device=dev)
        self.y16 = torch.empty((16, self.rows), dtype=torch.float32, device=dev)
        self.launches_per_step = 4  # encode, decode, gemv b1, gemv b16 (+2 memsets)
        self.ev = {"encode": [], "decode": [], "gemv1": [], "gemv16": []}

    def bytes_decoded(self):
        return self.n * 256

    def bytes_encoded(self):
        return self.n * 256

    def _t(self, key, fn, record):
        if record:
            a, b = _events(self.torch)
            a.record()
        fn()
        if record:
            b.record()
            self.ev[key].append((a, b))

    def step(self, record=False):
        e = self.ecco
        self._t("encode", lambda: e.encode(self.w, self.tables, out=self.blocks), record)
        self._t("decode", lambda: e.decode(self.blocks, self.tables, out=self.out), record)
        self._t("gemv1", lambda: e.decode_gemv(self.blocks, self.tables, self.rows, self.cols, self.x1, out=self.y1), record)
        self._t("gemv16", lambda: e.decode_gemv(self.blocks, self.tables, self.rows, self.cols, self.x16, out=self.y16), record)

    def dominant(self):
        self.torch.cuda.synchronize()
        return "decode_kernel", self.n * 320, [a.elapsed_time(b) for a, b in self.ev["decode"]]

    def per_op(self):
        self.torch.cuda.synchronize()
        out = {}
        byts = {"encode": self.n * 320, "decode": self.n * 320,
                "gemv1": self.n * 64 + self.cols * 2 + self.rows * 4,
                "gemv16": self.n * 64 + 16 * self.cols * 2 + 16 * self.rows * 4}
        for k, evs in self.ev.items():
            ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
            out[k] = {"ms": ms, "algorithmic_bytes": byts[k], "GB_s": byts[k] / ms / 1e6}
        return out

    def e2e_setup(self):
        self.hw = self.w.cpu().pin_memory()
        self.hx = self.x1.cpu().pin_memory()
        self.hy = self.torch.empty((self.n, 128), dtype=self.torch.bfloat16).pin_memory()
        self.hy1 = self.torch.empty((1, self.rows), dtype=self.torch.float32).pin_memory()
        self.dw = self.torch.empty_like(self.w)
        self.h2d = self.hw.numel() * 2 + self.hx.numel() * 2
        self.d2h = self.hy.numel() * 2 + self.hy1.numel() * 4

    def e2e_step(self):
        e = self.ecco
        self.dw.copy_(self.hw, non_blocking=True)
        self.x1.copy_(self.hx, non_blocking=True)
        e.encode(self.dw, self.tables, out=self.blocks)
        e.decode(self.blocks, self.tables, out=self.out)
        e.decode_gemv(self.blocks, self.tables, self.rows, self.cols, self.x1, out=self.y1)
        e.decode_gemv(self.blocks, self.tables, self.rows, self.cols, self.x16, out=self.y16)
        self.hy.copy_(self.out, non_blocking=True)
        self.hy1.copy_(self.y1, non_blocking=True)

    def cpu_sample(self, frac):
        import workloads as W
        n = max(64, int(self.n * frac))
        xb = W.bf16_bits(self.w.view(-1, 128)[:n])
        return {"enc": [(self.tables.blob, xb)], "dec": [(self.tables.blob, self.blocks[:n].cpu().numpy())],
                "bytes": 2 * n * 256, "what": f"encode {n} groups + decode {n} blocks (1/{round(1 / frac)} of a step, GEMV not sampled)"}


class ModelWorkload(Workload):
    """All 224 weight tensors of a 32-layer Llama-3-8B-shaped model: encode the
    whole set, decode the whole set (one multi-segment launch per 64 tensors)."""
    name = "model"
    layers = 32  # bench.py --layers: fewer only for profiling captures
    desc = ("Llama-3-8B-shaped weights, 32 layers x {q,k,v,o 4096/1024 x 4096; gate,up 14336 x 4096; "
            "down 4096 x 14336}, Student-t(5) x 0.02, per-tensor tables: whole-model encode + decode")

    def __init__(self, dev, seed_offset=0):
        import torch
        import workloads as W
        import entropy_coded_kv_b200 as ecco
        self.torch, self.ecco, self.dev = torch, ecco, dev
        self.w, self.tables = [], []
        self.per_layer = len(W.C4_SHAPES)
        self.layers = min(self.layers, W.C4_LAYERS)
        for layer in range(self.layers):
            for name, _, _ in W.C4_SHAPES:
                t = W.c4_tensor(layer, name, device=dev, seed=4 + seed_offset)
                self.w.append(t)
                self.tables.append(ecco.Tables(ecco.learn_tables(t, seed=layer), dev))  # GPU learner
        self.blocks = [torch.empty((t.numel() // 128, 64), dtype=torch.uint8, device=dev) for t in self.w]
        self.out = [torch.empty_like(t) for t in self.w]
        self.n = sum(t.numel() // 128 for t in self.w)
        self.enc = [ecco.Seg(tb, t, b) for tb, t, b in zip(self.tables, self.w, self.blocks)]
        self.dec = [ecco.Seg(tb, b, o.view(-1, 128)) for tb, b, o in zip(self.tables, self.blocks, self.out)]
        st = ecco.new_stats(dev)
        ecco.encode_multi(self.enc, st)
        self.stats, self.n_tensors = ecco.read_stats(st), len(self.w)
        self.launches_per_step = 2 * ((len(self.w) + 63) // 64)
        self.ev = {"encode": [], "decode": []}

    def bytes_decoded(self):
        return self.n * 256

    def bytes_encoded(self):
        return self.n * 256

    def cpu_frac(self):
        return 1.0 / 1000

    def step(self, record=False):
        for key, fn in (("encode", lambda: self.ecco.encode_multi(self.enc)),
                        ("decode", lambda: self.ecco.decode_multi(self.dec))):
            if record:
                a, b = _events(self.torch)
                a.record()
            fn()
            if record:
                b.record()
                self.ev[key].append((a, b))

    def dominant(self):
        self.torch.cuda.synchronize()
        return "decode_kernel (multi-segment)", self.n * 320, [a.elapsed_time(b) for a, b in self.ev["decode"]]

    def per_op(self):
        self.torch.cuda.synchronize()
        out = {}
        for k, evs in self.ev.items():
            ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
            out[k] = {"ms": ms, "algorithmic_bytes": self.n * 320, "GB_s": self.n * 320 / ms / 1e6,
                      "launches": (len(self.w) + 63) // 64}
        return out

    def e2e_setup(self):
        """Per layer: H2D of its 7 bf16 weights, encode_multi + decode_multi of
        the layer, D2H of its blocks and decoded weights."""
        torch, e = self.torch, self.ecco
        self.h_w = [t.cpu().pin_memory() for t in self.w]
        self.d_w = [torch.empty_like(t) for t in self.w]
        k = self.per_layer
        enc = [e.Seg(tb, dw, b) for tb, dw, b in zip(self.tables, self.d_w, self.blocks)]
        layers = []
        for i in range(0, len(self.w), k):
            layers.append(([(self.h_w[j], self.d_w[j]) for j in range(i, i + k)],
                           (lambda a, b: lambda: (e.encode_multi(a), e.decode_multi(b)))(enc[i:i + k],
                                                                                      self.dec[i:i + k]),
                           self.blocks[i:i + k] + self.out[i:i + k]))
        self.stream = LayerStream(torch, self.dev, layers)
        self.h2d, self.d2h = self.stream.h2d, self.stream.d2h
        self.api = ("entropy_coded_kv_b200.encode_multi/decode_multi (C ABI), streamed per layer: H2D of the "
                    "layer's bf16 weights from pinned host memory, D2H of its blocks and decoded weights")

    def e2e_step(self):
        self.stream.step()

    def cpu_sample(self, frac):
        import workloads as W
        enc, dec, nb = [], [], 0
        for t, tb, b in zip(self.w, self.tables, self.blocks):
            k = max(8, int(t.numel() // 128 * frac))
            enc.append((tb.blob, W.bf16_bits(t.view(-1, 128)[:k])))
            dec.append((tb.blob, b[:k].cpu().numpy()))
            nb += k
        return {"enc": enc, "dec": dec, "bytes": 2 * nb * 256,
                "what": f"encode + decode of the first {nb} groups across all 224 tensors (1/{round(1 / frac)} of a step)"}


class LongCtxWorkload(Workload):
    """32 layers x K,V x [1, 8, 131072, 128] KV cache: decode the whole cache
    and append one token per layer (K and V), per step."""
    name = "longctx"
    layers = 32  # bench.py --layers: fewer only for profiling captures
    desc = ("long-context KV cache, 32 layers x K,V x [1, 8, 131072, 128] bf16 (17.2 GB), per-layer K/V "
            "tables from [1, 8, 4096, 128] calibration samples: decode the whole cache + append one token "
            "per layer (512 groups)")
    S = 131072

    def __init__(self, dev, seed_offset=0):
        import torch
        import workloads as W
        import entropy_coded_kv_b200 as ecco
        self.torch, self.ecco, self.dev = torch, ecco, dev
        self.caches, self.tables = [], []
        for layer in range(min(self.layers, 32)):
            K, V = W.c5_layer(layer, device=dev, seed=5 + seed_offset)
            Kc, Vc = W.c5_calibration(layer, device=dev, seed=105 + seed_offset)
            self.caches += [K, V]
            self.tables += [ecco.Tables(ecco.learn_tables(c, seed=layer), dev) for c in (Kc, Vc)]  # GPU learner
            del Kc, Vc
        self.blocks = [torch.empty((c.numel() // 128, 64), dtype=torch.uint8, device=dev) for c in self.caches]
        st = ecco.new_stats(dev)
        ecco.encode_multi([ecco.Seg(tb, c, b) for tb, c, b in zip(self.tables, self.caches, self.blocks)], st)
        self.stats, self.n_tensors = ecco.read_stats(st), len(self.caches)
        self.out = [torch.empty_like(c) for c in self.caches]
        self.new = [c.view(8, self.S, 128)[:, self.S - 1:].contiguous() for c in self.caches]
        app = ecco.kv_append_desc(8, 1, self.S, self.S - 1)
        # checked and marshalled once: a step only passes the prepared segments
        self.app = ecco.prepare_encode([ecco.Seg(tb, nw, b, app) for tb, nw, b in zip(self.tables, self.new, self.blocks)])
        self.dec_segs = [ecco.Seg(tb, b, o.view(-1, 128)) for tb, b, o in zip(self.tables, self.blocks, self.out)]
        self.dec = ecco.prepare_decode(self.dec_segs)
        self.n = sum(c.numel() // 128 for c in self.caches)
        self.launches_per_step = 2
        self.ev = {"encode": [], "decode": []}

    def bytes_decoded(self):
        return self.n * 256

    def bytes_encoded(self):
        return len(self.new) * 8 * 256

    def cpu_frac(self):
        return 1.0 / 1000

    def step(self, record=False):
        for key, fn in (("encode", lambda: self.ecco.encode_multi(self.app)),
                        ("decode", lambda: self.ecco.decode_multi(self.dec))):
            if record:
                a, b = _events(self.torch)
                a.record()
            fn()
            if record:
                b.record()
                self.ev[key].append((a, b))

    def dominant(self):
        self.torch.cuda.synchronize()
        return "decode_kernel (multi-segment)", self.n * 320, [a.elapsed_time(b) for a, b in self.ev["decode"]]

    def per_op(self):
        self.torch.cuda.synchronize()
        nb = {"encode": len(self.new) * 8 * 320, "decode": self.n * 320}
        return {k: {"ms": statistics.mean(a.elapsed_time(b) for a, b in evs), "algorithmic_bytes": nb[k],
                    "GB_s": nb[k] / statistics.mean(a.elapsed_time(b) for a, b in evs) / 1e6}
                for k, evs in self.ev.items()}

    def e2e_setup(self):
        """Per layer: H2D of its compressed K and V caches and of the new
        token, the append and the decode of the layer, D2H of the decoded K
        and V."""
        torch, e = self.torch, self.ecco
        self.h_blocks = [b.cpu().pin_memory() for b in self.blocks]
        self.h_new = [t.cpu().pin_memory() for t in self.new]
        self.d_new = [torch.empty_like(t) for t in self.new]
        app = e.kv_append_desc(8, 1, self.S, self.S - 1)
        e2e_app = [e.Seg(tb, dn, b, app) for tb, dn, b in zip(self.tables, self.d_new, self.blocks)]
        layers = []
        for i in range(0, len(self.caches), 2):
            ins = [(self.h_blocks[j], self.blocks[j]) for j in (i, i + 1)] + \
                  [(self.h_new[j], self.d_new[j]) for j in (i, i + 1)]
            layers.append((ins, (lambda a, b: lambda: (e.encode_multi(a), e.decode_multi(b)))(
                               e.prepare_encode(e2e_app[i:i + 2]), e.prepare_decode(self.dec_segs[i:i + 2])),
                           self.out[i:i + 2]))
        self.stream = LayerStream(torch, self.dev, layers)
        self.h2d, self.d2h = self.stream.h2d, self.stream.d2h
        self.launches_e2e = 2 * len(layers)
        self.api = ("entropy_coded_kv_b200.encode_multi/decode_multi (C ABI), streamed per layer: H2D of the "
                    "layer's compressed K, V and new token from pinned host memory, D2H of its decoded K and V")

    def e2e_step(self):
        self.stream.step()

    def cpu_sample(self, frac):
        import workloads as W
        enc = [(tb.blob, W.bf16_bits(nw.view(-1, 128))) for tb, nw in zip(self.tables, self.new)]
        dec, nb = [], 0
        for tb, b in zip(self.tables, self.blocks):
            k = max(8, int(b.shape[0] * frac))
            dec.append((tb.blob, b[:k].cpu().numpy()))
            nb += k
        return {"enc": enc, "dec": dec, "bytes": nb * 256 + len(self.new) * 8 * 256,
                "what": f"the per-step append (512 groups) + decode of {nb} blocks (1/{round(1 / frac)} of the cache)"}


class AttnWorkload(Workload):
    """One decode step of attention over a compressed KV cache: append the new
    token's K and V, then attention of 32 query heads (group 4) over all 4096
    tokens, the blocks decoded inside the attention kernel."""
    name = "attn"
    B, H, S, D, G = 8, 8, 4096, 128, 4
    path = "staged"  # or "fused": the single kernel that decodes inside the attention

    @staticmethod
    def describe(path):
        how = ("staged decode+attention over all 4096 tokens (block decoder into a workspace scratch, then "
               "the split kernel)" if path == "staged" else
               "fused decode+attention over all 4096 tokens (one kernel decodes and attends)")
        return ("decode-phase attention over a compressed Llama-3-8B-shaped layer KV cache: K, V "
                "[8, 8, 4096, 128] as 64-byte blocks, 32 query heads (group 4); a step appends one "
                "token's K and V (128 groups) and runs " + how)

    def __init__(self, dev, seed_offset=0):
        import torch
        import workloads as W
        import entropy_coded_kv_b200 as ecco
        from entropy_coded_kv_b200.calib import learn_tables
        self.torch, self.ecco, self.dev = torch, ecco, dev
        self.desc = self.describe(self.path)
        K, V = W.c2_kv(device=dev, seed=1 + seed_offset)
        Kc, Vc = W.c2_calibration(device=dev, seed=2 + seed_offset)
        self.tables = [ecco.Tables(learn_tables(Kc, seed=0), dev), ecco.Tables(learn_tables(Vc, seed=0), dev)]
        self.rows = self.B * self.H
        self.n = self.rows * self.S
        st = ecco.new_stats(dev)
        self.blocks = [ecco.encode(K, self.tables[0], stats=st).view(self.B, self.H, self.S, 64),
                       ecco.encode(V, self.tables[1], stats=st).view(self.B, self.H, self.S, 64)]
        self.stats, self.n_tensors = ecco.read_stats(st), 2
        self.new = [K.view(self.rows, self.S, self.D)[:, self.S - 1:].contiguous(),
                    V.view(self.rows, self.S, self.D)[:, self.S - 1:].contiguous()]
        self.append = ecco.kv_append_desc(self.rows, 1, self.S, self.S - 1)
        self.app = [ecco.Seg(self.tables[i], self.new[i], self.blocks[i], self.append) for i in range(2)]
        g = torch.Generator(device=dev).manual_seed(77 + seed_offset)
        self.q = torch.randn(self.B, self.H * self.G, self.D, generator=g, device=dev).to(torch.bfloat16)
        self.out = torch.empty(self.B, self.H * self.G, self.D, dtype=torch.float32, device=dev)
        staged = self.path == "staged"
        ws_bytes = ecco.attention_staged_workspace_bytes if staged else ecco.attention_workspace_bytes
        self.ws = torch.empty(ws_bytes(self.B, self.H, self.G, self.S), dtype=torch.uint8, device=dev)
        self.attend = ecco.decode_attention_staged if staged else ecco.decode_attention
        self.scale = 1.0 / self.D ** 0.5
        # append (one multi-segment launch); staged, one chunk: decode (K and V in one launch) and the
        # split kernel; fused: the split kernel; then the merge
        self.launches_per_step = 4 if staged else 3
        self.api = (f"entropy_coded_kv_b200.encode_multi/{self.attend.__name__} (C ABI) with pinned host "
                    "buffers")
        self.att_ms = []

    def bytes_decoded(self):  # bf16 K and V bytes the step decodes
        return 2 * self.n * 256

    def bytes_encoded(self):
        return 2 * self.rows * 256

    def cpu_frac(self):
        return 1.0 / 64

    def _attend(self, q):
        return self.attend(self.blocks[0], self.blocks[1], self.tables[0], self.tables[1], q, self.S, self.scale,
                           out=self.out, workspace=self.ws)

    def step(self, record=False):
        self.ecco.encode_multi(self.app)
        if record:
            a, b = _events(self.torch)
            a.record()
        self._attend(self.q)
        if record:
            b.record()
            self.att_ms.append((a, b))

    def dominant(self):
        """Algorithmic bytes: compressed K and V read once, q read, output written."""
        self.torch.cuda.synchronize()
        ms = [a.elapsed_time(b) for a, b in self.att_ms]
        nbytes = 2 * self.n * 64 + self.q.numel() * 2 + self.out.numel() * 4
        kernels = "decode_kernel+attn_split_kernel+attn_merge_kernel" if self.path == "staged" else \
            "attn_split_kernel+attn_merge_kernel"
        return kernels, nbytes, ms

    def e2e_setup(self):
        torch = self.torch
        self.h_new = [t.cpu().pin_memory() for t in self.new]
        self.h_q = self.q.cpu().pin_memory()
        self.h_out = torch.empty(self.out.shape, dtype=torch.float32).pin_memory()
        self.d_new = [torch.empty_like(t) for t in self.new]
        self.d_q = torch.empty_like(self.q)
        self.e2e_app = [self.ecco.Seg(self.tables[i], self.d_new[i], self.blocks[i], self.append) for i in range(2)]
        self.h2d = sum(t.numel() * t.element_size() for t in self.h_new) + self.h_q.numel() * 2
        self.d2h = self.h_out.numel() * 4

    def e2e_step(self):
        for i in range(2):
            self.d_new[i].copy_(self.h_new[i], non_blocking=True)
        self.d_q.copy_(self.h_q, non_blocking=True)
        self.ecco.encode_multi(self.e2e_app)
        self._attend(self.d_q)
        self.h_out.copy_(self.out, non_blocking=True)

    def cpu_sample(self, frac):
        import workloads as W
        pairs = max(1, int(self.rows * frac))
        kb = [self.blocks[i].view(self.rows, self.S, 64)[:pairs].cpu().numpy() for i in range(2)]
        qb = W.bf16_bits(self.q.view(self.rows, self.G, self.D)[:pairs])
        xs = [W.bf16_bits(self.new[i][:pairs].reshape(-1, 128)) for i in range(2)]
        blobs = [t.blob for t in self.tables]
        return {"enc": [(blobs[i], xs[i]) for i in range(2)], "dec": [],
                "attn": (blobs, kb, qb, self.S, self.scale),
                "bytes": 2 * pairs * self.S * 256 + 2 * pairs * 256,
                "what": f"append + attention for {pairs} of {self.rows} (batch, KV head) pairs "
                        f"({2 * pairs * self.S} blocks decoded)"}


class SelectWorkload(Workload):
    """Pattern-selection study on the KV cache: a step encodes K and V of the
    [8, 8, 4096, 128] layer with full-MSE pattern selection (64 patterns);
    setup also times and scores min/max and the 16-pattern variants."""
    name = "select"
    desc = ("KV cache [8, 8, 4096, 128] K and V: encode with full-MSE pattern selection over 64 "
            "patterns (524,288 groups); quality of min/max vs full-MSE selection, 64 and 16 patterns")
    B, H, S, D = 8, 8, 4096, 128

    def __init__(self, dev, seed_offset=0):
        import torch
        import workloads as W
        import entropy_coded_kv_b200 as ecco
        from entropy_coded_kv_b200 import _lib
        from entropy_coded_kv_b200.calib import learn_tables
        self.torch, self.ecco, self.dev, self._lib = torch, ecco, dev, _lib
        K, V = W.c2_kv(device=dev, seed=1 + seed_offset)
        Kc, Vc = W.c2_calibration(device=dev, seed=2 + seed_offset)
        self.x = [K, V]
        self.n = K.numel() // 128
        self.tabs = {64: [ecco.Tables(learn_tables(c, seed=0), dev) for c in (Kc, Vc)],
                     16: [ecco.Tables(learn_tables(c, seed=0, npat=16), dev) for c in (Kc, Vc)]}
        self.blocks = [torch.empty((self.n, 64), dtype=torch.uint8, device=dev) for _ in range(2)]
        self.launches_per_step = 2
        self.enc_ms = []
        self.quality = self._study()

    def _study(self):
        torch, ecco = self.torch, self.ecco
        out, chosen = {}, {}
        for npat in (64, 16):
            for sel, sname in ((self._lib.SELECT_MINMAX, "minmax"), (self._lib.SELECT_MSE, "mse")):
                err = ref = 0.0
                ps = []
                for i in range(2):
                    t = self.tabs[npat][i]
                    ecco.encode(self.x[i], t, out=self.blocks[i], select=sel, n_patterns=npat)
                    torch.cuda.synchronize()
                    a, b = _events(torch)
                    a.record()
                    ecco.encode(self.x[i], t, out=self.blocks[i], select=sel, n_patterns=npat)
                    b.record()
                    y = ecco.decode(self.blocks[i], t).float().view_as(self.x[i])
                    xf = self.x[i].float()
                    err += float(((y - xf) ** 2).sum())
                    ref += float((xf ** 2).sum())
                    ps.append((self.blocks[i][:, 1] & 63).clone())
                    torch.cuda.synchronize()
                    ms = a.elapsed_time(b)
                    out.setdefault(f"{sname}{npat}", {"encode_GBps": []})["encode_GBps"].append(
                        round(self.n * 256 / (ms * 1e-3) / 1e9, 1))
                out[f"{sname}{npat}"]["rel_mse"] = err / ref
                chosen[(sname, npat)] = torch.cat(ps)
        for npat in (64, 16):
            diff = (chosen[("minmax", npat)] != chosen[("mse", npat)]).float().mean().item()
            out[f"minmax{npat}"]["pattern_differs_from_mse"] = round(diff, 4)
        return out

    def bytes_encoded(self):
        return 2 * self.n * 256

    def cpu_frac(self):
        return 1.0 / 512

    def step(self, record=False):
        if record:
            a, b = _events(self.torch)
            a.record()
        for i in range(2):
            self.ecco.encode(self.x[i], self.tabs[64][i], out=self.blocks[i], select=self._lib.SELECT_MSE)
        if record:
            b.record()
            self.enc_ms.append((a, b))

    def dominant(self):
        self.torch.cuda.synchronize()
        return "encode_kernel<.,SEL=1>", 2 * self.n * 320, [a.elapsed_time(b) for a, b in self.enc_ms]

    def per_op(self):
        return {"selection_study": self.quality}

    def e2e_setup(self):
        torch = self.torch
        self.hx = [t.cpu().pin_memory() for t in self.x]
        self.hb = [torch.empty((self.n, 64), dtype=torch.uint8).pin_memory() for _ in range(2)]
        self.dx = [torch.empty_like(t) for t in self.x]
        self.h2d = sum(t.numel() * 2 for t in self.hx)
        self.d2h = sum(t.numel() for t in self.hb)

    def e2e_step(self):
        for i in range(2):
            self.dx[i].copy_(self.hx[i], non_blocking=True)
            self.ecco.encode(self.dx[i], self.tabs[64][i], out=self.blocks[i], select=self._lib.SELECT_MSE)
            self.hb[i].copy_(self.blocks[i], non_blocking=True)

    def cpu_sample(self, frac):
        import workloads as W
        k = max(64, int(self.n * frac))
        xs = [W.bf16_bits(self.x[i].view(-1, 128)[:k]) for i in range(2)]
        return {"enc": [(self.tabs[64][i].blob, xs[i]) for i in range(2)], "dec": [],
                "select": 1, "bytes": 2 * k * 256,
                "what": f"full-MSE encode of {2 * k} groups (1/{round(1 / frac)} of a step)"}


class ActWorkload(Workload):
    """Activation format: [8192, 4096] bf16 hidden states (Llama-3-8B width) in
    64-value groups; a step encodes and decodes all 524,288 groups."""
    name = "act"
    desc = ("activations [8192, 4096] bf16 (channel-outlier hidden states) in the 2x format: "
            "64-value groups, 524,288 blocks; encode + decode")
    T, D, GA = 8192, 4096, 64

    def __init__(self, dev, seed_offset=0):
        import torch
        import workloads as W
        import entropy_coded_kv_b200 as ecco
        from entropy_coded_kv_b200.calib import learn_tables
        self.torch, self.ecco, self.dev = torch, ecco, dev
        self.x = W.hidden_states(self.T, self.D, seed=6 + seed_offset, device=dev)
        self.tables = ecco.Tables(learn_tables(W.hidden_states(2048, self.D, seed=61 + seed_offset),
                                               seed=0, group=self.GA), dev)
        self.n = self.x.numel() // self.GA
        st = ecco.new_stats(dev)
        self.blocks = ecco.encode_act(self.x, self.tables, stats=st)
        self.stats, self.group = ecco.read_stats(st), self.GA
        self.out = torch.empty((self.n, self.GA), dtype=torch.bfloat16, device=dev)
        self.launches_per_step = 2
        self.dec_ms = []

    def bytes_decoded(self):
        return self.n * self.GA * 2

    def bytes_encoded(self):
        return self.n * self.GA * 2

    def cpu_frac(self):
        return 1.0 / 64

    def step(self, record=False):
        self.ecco.encode_act(self.x, self.tables, out=self.blocks)
        if record:
            a, b = _events(self.torch)
            a.record()
        self.ecco.decode_act(self.blocks, self.tables, out=self.out)
        if record:
            b.record()
            self.dec_ms.append((a, b))

    def dominant(self):
        self.torch.cuda.synchronize()
        return "decode_kernel<G=64>", self.n * (64 + 128), [a.elapsed_time(b) for a, b in self.dec_ms]

    def e2e_setup(self):
        torch = self.torch
        self.hx = self.x.cpu().pin_memory()
        self.hy = torch.empty((self.n, self.GA), dtype=torch.bfloat16).pin_memory()
        self.dx = torch.empty_like(self.x)
        self.h2d, self.d2h = self.hx.numel() * 2, self.hy.numel() * 2
        self.api = "entropy_coded_kv_b200.encode_act/decode_act (C ABI) with pinned host buffers"

    def e2e_step(self):
        self.dx.copy_(self.hx, non_blocking=True)
        self.ecco.encode_act(self.dx, self.tables, out=self.blocks)
        self.ecco.decode_act(self.blocks, self.tables, out=self.out)
        self.hy.copy_(self.out, non_blocking=True)

    def cpu_sample(self, frac):
        import workloads as W
        k = max(64, int(self.n * frac))
        xb = W.bf16_bits(self.x.view(-1, self.GA)[:k])
        bl = self.blocks[:k].cpu().numpy()
        return {"enc": [(self.tables.blob, xb)], "dec": [(self.tables.blob, bl)], "gs": self.GA,
                "bytes": 2 * k * self.GA * 2,
                "what": f"encode + decode of {k} activation groups (1/{round(1 / frac)} of a step)"}


WORKLOADS = {"act": ActWorkload, "kv": KVWorkload, "c1": C1Workload, "mlp": MLPWorkload, "model": ModelWorkload,
             "longctx": LongCtxWorkload, "attn": AttnWorkload, "select": SelectWorkload}


# ------------------------------------------------------------------ host-only samples (reference arm)
def host_sample(name):
    """A bounded sample of workload `name` built on the host alone, for the
    oracle arm: inputs from `workloads` on the CPU (the workload's
    distribution and seeds, at a reduced size where the full one would take
    minutes to generate or run), tables from the host learner
    (entropy_coded_kv_b200.calib, numpy) on a small calibration sample, blocks
    from the oracle's own encoder.  No device and no libecco_b200.so."""
    import numpy as np
    import torch
    import oracle
    import workloads as W
    from entropy_coded_kv_b200.calib import learn_tables

    def bits(t):
        return W.bf16_bits(t)

    def enc(blob, xb, gs=128):
        return oracle.encode(blob, xb, nthreads=os.cpu_count() or 1, gs=gs)[0]

    if name == "c1":
        x = W.c1_matrix(seed=0)
        blob = learn_tables(x)
        xb = bits(x)
        return {"enc": [(blob, xb)], "dec": [(blob, enc(blob, xb))], "bytes": 2 * 2048 * 256,
                "what": "the whole step (encode 2048 groups + decode 2048 blocks)"}
    if name in ("kv", "select"):
        K, V = W.c2_kv(seed=1)
        cal = W.kv_cache((1, 8, 256, 128), 2)
        blobs = [learn_tables(cal[0], seed=0), learn_tables(cal[1], seed=0)]
        if name == "select":
            k = 2048
            xs = [bits(t.reshape(-1, 128)[:k]) for t in (K, V)]
            return {"enc": list(zip(blobs, xs)), "dec": [], "select": 1, "bytes": 2 * k * 256,
                    "what": f"full-MSE encode of {2 * k} groups (1/{524288 // k} of a step)"}
        new = [bits(t.reshape(64, 4096, 128)[:, 4032:]) for t in (K, V)]
        dec = [(b, enc(b, bits(t))) for b, t in zip(blobs, (K, V))]
        return {"enc": list(zip(blobs, new)), "dec": dec, "bytes": 2 * 524288 * 256 + 2 * 8192 * 256,
                "what": "the whole step (encode 8,192 groups of K and of V + decode 524,288 blocks of each)"}
    if name == "mlp":
        g = W._gen(3, "cpu")
        w = (W.student_t((896, 4096), 5, g, "cpu") * 0.02).to(dtype=torch.bfloat16)
        blob = learn_tables(w[:64])
        xb = bits(w)
        n = xb.size // 128
        return {"enc": [(blob, xb)], "dec": [(blob, enc(blob, xb))], "bytes": 2 * n * 256,
                "what": f"encode + decode of {n} groups (896 of 14,336 rows; GEMV not sampled)"}
    if name == "model":
        encs, decs, nb = [], [], 0
        shape_blob = {}
        for layer in range(W.C4_LAYERS):
            for i, (sh, rows, cols) in enumerate(W.C4_SHAPES):
                g = W._gen(4 * 1000 + layer * len(W.C4_SHAPES) + i, "cpu")
                k = max(8, rows * cols // 128 // 1000)
                t = (W.student_t((k, 128), 5, g, "cpu") * 0.02).to(dtype=torch.bfloat16)
                if sh not in shape_blob:
                    cal = (W.student_t((2048, 128), 5, W._gen(40 + i, "cpu"), "cpu") * 0.02).to(dtype=torch.bfloat16)
                    shape_blob[sh] = learn_tables(cal)
                blob, xb = shape_blob[sh], bits(t)
                encs.append((blob, xb))
                decs.append((blob, enc(blob, xb)))
                nb += k
        return {"enc": encs, "dec": decs, "bytes": 2 * nb * 256,
                "what": f"encode + decode of {nb} groups across all 224 tensors (1/1000 of each; one table set "
                        f"per tensor shape)"}
    if name == "longctx":
        encs, decs, nb = [], [], 0
        tok = 1311  # ~1% of the 131,072 tokens of every head
        for layer in range(32):
            kv = W.kv_cache((1, 8, tok, 128), 5 * 1000 + layer)
            cal = W.kv_cache((1, 8, 256, 128), 105 * 1000 + layer)
            for t, c in zip(kv, cal):
                blob = learn_tables(c, seed=layer)
                xb = bits(t).reshape(8, tok, 128)
                encs.append((blob, np.ascontiguousarray(xb[:, -1])))
                decs.append((blob, enc(blob, xb.reshape(-1, 128))))
                nb += 8 * tok
        return {"enc": encs, "dec": decs, "bytes": nb * 256 + 512 * 256,
                "what": f"the per-step append (512 groups) + decode of {nb} blocks ({tok} of 131,072 tokens of "
                        f"every head of all 64 caches)"}
    if name == "attn":
        K, V = W.kv_cache((1, 1, 4096, 128), 1)
        cal = W.kv_cache((1, 8, 256, 128), 2)
        blobs = [learn_tables(cal[0], seed=0), learn_tables(cal[1], seed=0)]
        kb = [enc(b, bits(t)).reshape(1, 4096, 64) for b, t in zip(blobs, (K, V))]
        q = torch.randn(1, 4, 128, generator=W._gen(77, "cpu")).to(torch.bfloat16)
        xs = [bits(t.reshape(4096, 128)[-1:]) for t in (K, V)]
        return {"enc": list(zip(blobs, xs)), "dec": [], "attn": (blobs, kb, bits(q), 4096, 128 ** -0.5),
                "bytes": 2 * 4096 * 256 + 2 * 256,
                "what": "append + attention for 1 of 64 (batch, KV head) pairs (8,192 blocks decoded)"}
    if name == "act":
        x = W.hidden_states(128, 4096, seed=6)
        blob = learn_tables(W.hidden_states(32, 4096, seed=61), seed=0, group=64)
        xb = bits(x)
        n = xb.size // 64
        return {"enc": [(blob, xb)], "dec": [(blob, enc(blob, xb, 64))], "gs": 64, "bytes": 2 * n * 128,
                "what": f"encode + decode of {n} activation groups (128 of 8,192 tokens)"}
    raise KeyError(name)


# ------------------------------------------------------------------ CPU oracle timing
def time_oracle(sample, nthreads):
    import oracle
    t0 = time.perf_counter()
    gs = sample.get("gs", 128)
    for blob, xb in sample["enc"]:
        oracle.encode(blob, xb, nthreads=nthreads, select=sample.get("select", 0), gs=gs)
    for blob, bl in sample["dec"]:
        oracle.decode(blob, bl, nthreads=nthreads, gs=gs)
    if "attn" in sample:
        (kt, vt), (kb, vb), qb, S, scale = sample["attn"]
        n = kb.shape[0]
        oracle.attention(kt, vt, kb.reshape(n, 1, S, 64), vb.reshape(n, 1, S, 64), qb, S, scale, nthreads=nthreads)
    return time.perf_counter() - t0


def cpu_baseline(wl, target_s):
    """The oracle as it stands, on a bounded sample of the step, repeated until
    about target_s seconds of host work have been timed."""
    cores = os.cpu_count() or 1
    frac = wl.cpu_frac()
    sample = wl.cpu_sample(frac)
    dt = time_oracle(sample, cores)
    reps, total = 1, dt
    while total < target_s and reps < 1000:
        total += time_oracle(sample, cores)
        reps += 1
    one = time_oracle(sample, 1)  # the same sample on one host thread, once
    return {"value": sample["bytes"] * reps / total / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"{sample['what']}, {reps} repetitions", "seconds": round(total, 2),
            "value_1_thread": round(sample["bytes"] / one / 1e9, 4)}


# ------------------------------------------------------------------ main
def main():
    args = parse_args()
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        if args.impl == "ecco":  # one GPU per rank, bound before the first collective
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=300))

    if args.impl == "reference":
        if rank == 0:
            run_reference(args, world)
        if world > 1:
            dist.destroy_process_group()
        return

    from entropy_coded_kv_b200.build import build
    if rank == 0 or world == 1:
        build()
    if world > 1:
        dist.barrier()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    AttnWorkload.path = args.attention
    KVWorkload.speculative = args.decoder == "speculative"
    ModelWorkload.layers = LongCtxWorkload.layers = args.layers
    wl = WORKLOADS[args.workload](dev, seed_offset=0)
    if getattr(wl, "layers", 32) != 32:
        wl.desc = f"{wl.desc} [only {wl.layers} of 32 layers built]"
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    for _ in range(max(3, args.warmup)):
        wl.step()
        flush.fill_(1.0)
    torch.cuda.synchronize()

    clk = Clocks(dev)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clk.start()
    for i in range(args.steps):
        starts[i].record()
        wl.step(record=True)
        ends[i].record()
        flush.fill_(1.0)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = clk.stop()
    ms_total = sum(s.elapsed_time(e) for s, e in zip(starts, ends))
    t = torch.tensor([ms_total], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms_total = float(t.item())
    ms_step = ms_total / args.steps
    units = (wl.bytes_decoded() + wl.bytes_encoded()) * world
    value = units / (ms_step * 1e-3) / 1e9

    kname, kbytes, kms = wl.dominant()
    hbm, src = peaks()
    k_avg = statistics.mean(kms)
    achieved = kbytes / (k_avg * 1e-3) / 1e9
    roof = {"kernel": kname, "bound": "hbm", "achieved": round(achieved, 1), "peak": hbm,
            "unit": "GB/s", "frac": round(achieved / hbm, 4), "traffic": traffic_for(wl.name, kname),
            "peak_source": f"{src} (MEASURED_PEAKS.json hbm_gbs)" if src == "measured" else src,
            "algorithmic_bytes_per_launch": kbytes, "launch_ms": round(k_avg, 5)}

    e2e = None
    try:
        if not args.no_e2e:
            wl.e2e_setup()
    except NotImplementedError as why:
        e2e = {"value": None, "unit": "GB/s", "not_measured": str(why)}
        args.no_e2e = True
    if not args.no_e2e:
        for _ in range(2):
            wl.e2e_step()
        torch.cuda.synchronize()
        ks = max(3, min(args.steps, 10))
        a, b = _events(torch)
        a.record()
        for _ in range(ks):
            wl.e2e_step()
        b.record()
        torch.cuda.synchronize()
        ems = a.elapsed_time(b) / ks
        et = torch.tensor([ems], dtype=torch.float64, device=dev)
        if world > 1:
            dist.all_reduce(et, op=dist.ReduceOp.MAX)
        ems = float(et.item())
        e2e = {"value": round(units / (ems * 1e-3) / 1e9, 2), "unit": "GB/s", "ms_per_step": round(ems, 4),
               "h2d_bytes_per_step": wl.h2d, "d2h_bytes_per_step": wl.d2h,
               "api": getattr(wl, "api", "entropy_coded_kv_b200.encode/decode (C ABI) with pinned host buffers")}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl, args.cpu_seconds)

    ops = wl.per_op() if hasattr(wl, "per_op") else None
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": round(ms_step, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": wl.desc, "l2": "flushed between steps (256 MiB write outside the step events)",
                   "decoded_bf16_bytes_per_step": wl.bytes_decoded(),
                   "encoded_bf16_bytes_per_step": wl.bytes_encoded(),
                   "parallelism": f"replicas x{world} (independent blocks, no collective)"},
        "roofline": roof, "cpu_baseline": cpu, "e2e": e2e, "clocks": clocks,
        "gpu_launches": wl.launches_per_step * args.steps,
    }
    if ops:
        line["ops"] = ops
    summary = wl.stats_summary()
    if summary:
        line["stats"] = summary
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


# Sources each profiled kernel is built from: its DRAM traffic in
# profiles/traffic.json is used only while these files are unchanged.
KERNEL_SOURCES = {
    "decode_kernel": ["ecco_decode.cu", "ecco_block.cuh"],
    "decode_spec_kernel": ["ecco_decode_spec.cu", "ecco_block.cuh"],
    "decode_kernel<G=64>": ["ecco_decode.cu", "ecco_block.cuh"],
    "encode_kernel<.,SEL=1>": ["ecco_encode.cu", "ecco_bucket.cuh"],
    "decode_kernel+attn_split_kernel+attn_merge_kernel": ["ecco_attention.cu", "ecco_decode.cu", "ecco_block.cuh"],
    "attn_split_kernel+attn_merge_kernel": ["ecco_attention.cu", "ecco_block.cuh"],
}


def source_hash(files) -> str:
    """Hash of the files' code: comments and blank lines are left out, so a
    comment edit keeps a capture valid while any code change voids it."""
    import hashlib
    import re
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "entropy_coded_kv_b200", "csrc", f), encoding="utf-8") as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        code = "\n".join(line.rstrip() for line in text.splitlines() if line.strip())
        h.update(code.encode())
    return h.hexdigest()[:16]


def traffic_for(workload, kernel):
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    summary (profiles/traffic.json), or None when no capture matches or the
    kernel's sources changed since it was taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        entry = json.load(f).get("entries", {}).get(f"{workload}:{kernel}")
    if not entry:
        return None
    files = KERNEL_SOURCES.get(kernel.split(" ")[0], [])
    if not files or entry.get("source_hash") != source_hash(files):
        return None
    return entry.get("dram_bytes_per_launch")


def run_reference(args, world):
    """The CPU oracle as the reference arm: each step is a bounded sample of the
    workload (host_sample: built without a device or the product library),
    timed with the wall clock on the host cores."""
    cls = WORKLOADS[args.workload]
    desc = AttnWorkload.describe(args.attention) if cls is AttnWorkload else cls.desc
    cores = os.cpu_count() or 1
    sample = host_sample(args.workload)
    for _ in range(max(1, min(args.warmup, 2))):
        time_oracle(sample, cores)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        time_oracle(sample, cores)
    dt = (time.perf_counter() - t0) / args.steps
    v = sample["bytes"] / dt / 1e9
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(v, 4), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": desc, "sample": sample["what"]},
        "cpu_baseline": {"value": round(v, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": sample["what"]},
        "e2e": {"value": round(v, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)

if __name__ == "__main__":
    main()
