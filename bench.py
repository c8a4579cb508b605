#!/usr/bin/env python
"""Benchmark of the BLASST hot path on B200 (libblasst.so through its C ABI).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mine|reference]

Headline workload: GQA prefill with the Llama-3.1-8B attention shape (B=1,
Hq=32, Hkv=8, d=128, Lq=Lk=32768, causal, bf16) at the lambda that gives ~75%
block sparsity; one step = one prefill call.  Effective work per call counts
Q.K^T on every visited (tile, block) pair plus P.V on kept pairs, 2*128^3
FLOP each.  The same run also measures (the "sweep"): prefill at ~0/50/75%
sparsity and split-KV GQA decode (batch 32, Hq=32, Hkv=8, 32768-key cache,
16 splits) at ~0/50/75%, whose effective bytes are all K bytes + kept V bytes
+ q/o/lse.  Lambdas come from one calibration pass (decision-only kernel)
per workload: a pair is skipped iff its gap < ln(lambda), so the quantiles of
the gaps give the lambda for each target.

Inputs: seeded planted-direction generator ("blk" reading: planted logit +8,
5% heavy keys in 64-key runs, +2 local boost), bf16.  L2 is flushed (256 MiB
write) before every timed launch; timing uses CUDA events on the launching
stream.  The CPU baseline is the fp64 oracle timed on the host cores over a
bounded sample of query tiles of the same workload.

With N > 1 (torchrun), every rank runs an independent replica of the
workload on its own GPU (the problems are independent; no data-path
collective) and the timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "prefill eff. TFLOP/s & decode eff. HBM GB/s at 0/50/75% sparsity (1×B200)"
FLOP_PER_PAIR = 2 * 128 * 128 * 128
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# spec-sheet figures of one B200, for context beside the measured denominators
SPEC_PEAKS = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0}

PREFILL = dict(workload="prefill GQA 32K (Llama-3.1-8B attention shape)", B=1, Hq=32, Hkv=8, L=32768, d=128,
               causal=True, seed=2)
DECODE = dict(workload="decode GQA 32K cache, 16 splits", B=32, Hq=32, Hkv=8, Lk=32768, d=128, splits=16, seed=3)
MLA = dict(workload="MLA decode, 128 heads, 576/512 latent, 32K cache, 8 seeded splits", B=64, Hq=128, Lk=32768,
           splits=8, seed_splits=True, seed=5)
# 9 splits: what num_splits=-1 picks for this 128-row tile on 148 SMs (576 CTAs, just under two waves of two per SM)
MQA = dict(workload="decode MQA, 128 query heads on one KV head, 32K cache, 9 splits", B=64, Hq=128, Hkv=1,
           Lk=32768, d=128, splits=9, seed=9)
PREFILL_64K = dict(PREFILL, workload="prefill GQA 64K (Qwen3-8B-like attention shape)", L=65536, seed=4)
QUICK_PREFILL = dict(PREFILL, workload="prefill GQA 4K (quick)", L=4096)
QUICK_DECODE = dict(DECODE, workload="decode GQA 4K cache (quick)", B=4, Lk=4096)
# profiling size: inputs larger than L2 (126 MB) but a few GB at most on the device
MEDIUM_PREFILL = dict(PREFILL, workload="prefill GQA 16K (profiling size)", L=16384)
MEDIUM_DECODE = dict(DECODE, workload="decode GQA 32K cache, batch 8 (profiling size)", B=8)
MEDIUM_MLA = dict(MLA, workload="MLA decode, batch 16 (profiling size)", B=16)
QUICK_MLA = dict(MLA, workload="MLA decode (quick)", B=2, Lk=4096)
SIZES = {"full": (PREFILL, DECODE, MLA), "medium": (MEDIUM_PREFILL, MEDIUM_DECODE, MEDIUM_MLA),
         "quick": (QUICK_PREFILL, QUICK_DECODE, QUICK_MLA)}
TARGETS = (0.0, 0.5, 0.75)


def mqa_cfg(size, dcfg):
    """The 128-head MQA decode at the benchmark size, or a smaller batch at the other sizes."""
    return MQA if size == "full" else dict(MQA, B=max(2, MQA["B"] // 8), Lk=dcfg["Lk"])


# --------------------------------------------------------------------------- utils
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def load_profile_counters(kernel_key):
    """ncu counters of the benchmarked launch from the committed summary
    (profiles/traffic.json): {"dram_bytes_per_launch", "tensor_pipe_active_pct",
    ...}, or {} when none were taken for the current kernel build."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return d.get(kernel_key) or {}
    except Exception:
        return {}


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


class ClockSampler:
    """SM clock and clock-event (throttle) reasons, polled through NVML every
    few milliseconds while the timed region runs (read-only queries)."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, device_index):
        self.samples = []
        self.windows = []
        self.stop_flag = False
        self.h = None
        self.max_mhz = None
        try:
            import pynvml as nv
            import torch

            nv.nvmlInit()
            self.nv = nv
            props = torch.cuda.get_device_properties(device_index)
            try:
                bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
                self.h = nv.nvmlDeviceGetHandleByPciBusId(bus)
            except Exception:
                self.h = nv.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM)
        except Exception:
            self.h = None

    def start(self):
        if self.h is None:
            return
        self.t = threading.Thread(target=self._run, daemon=True)
        self.t.start()

    def _run(self):
        nv = self.nv
        while not self.stop_flag:
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                try:
                    r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                except Exception:
                    r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                self.samples.append((time.time(), mhz, r))
            except Exception:
                pass
            time.sleep(0.002)

    def mark(self, t0, t1):
        self.windows.append((t0, t1))

    def stop(self):
        self.stop_flag = True
        if self.h is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "source": "nvml unavailable"}
        self.t.join(timeout=2)
        inside = [s for s in self.samples if any(a <= s[0] <= b for a, b in self.windows)]
        use = inside or self.samples
        if not use:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0, "source": "nvml"}
        reasons = set()
        bits = 0
        for _, _, r in use:
            bits |= r
            for bit, name in self.REASONS.items():
                if r & bit:
                    reasons.add(name)
        mhz = sorted(s[1] for s in use)
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz, "sm_mhz_min": mhz[0],
                "sm_mhz_p90": mhz[int(0.9 * (len(mhz) - 1))], "reasons": sorted(reasons), "reason_bits": hex(bits),
                "samples": len(use), "in_timed_region": bool(inside), "source": "nvml"}


def to_dev(a, device):
    import numpy as np
    import torch

    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)


def to_pinned(a):
    import numpy as np
    import torch

    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).pin_memory()


# --------------------------------------------------------------------- workloads
def workload_name(kind, cfg):
    """The config name both bench arms print for a workload built on a base config."""
    if kind == "backward":
        return "fixed-mask backward, " + cfg["workload"]
    if kind == "decode_fp8":
        return cfg["workload"] + ", FP8 (e4m3) K/V cache"
    return cfg["workload"]


class Prefill:
    kind = "prefill"
    unit = "TFLOP/s"
    bound = "tensor"
    # end to end: device tensors filled from the host each step, read back each step, and private to a call
    e2e_in = ("q", "k", "v")
    e2e_out = ("o", "lse")
    e2e_private = ()

    def __init__(self, cfg, device):
        import synth

        self.cfg = cfg
        self.device = device
        c = cfg
        self.inp = synth.planted_prefill(c["B"], c["Hq"], c["Hkv"], c["L"], c["d"], seed=c["seed"], reading="blk")
        self.q, self.k, self.v = (to_dev(x, device) for x in (self.inp.q, self.inp.k, self.inp.v))
        import torch

        self.o = torch.empty_like(self.q)
        self.lse = torch.empty(self.q.shape[:3], dtype=torch.float32, device=device)
        import block_sparse_flashattention_tcgen05_b200 as bl

        self.bl = bl
        self.visited = bl.visited_pairs(c["B"], c["Hq"], c["Hkv"], c["L"], c["L"], True, False)
        self.launches = 1

    def calibrate(self):
        gaps, _, _ = self.bl.calibrate(self.q, self.k, scale=self.inp.scale, causal=True, mode="prefill")
        return gaps.cpu().numpy()

    def call(self, lam, stream=None):
        return self.bl.prefill(self.q, self.k, self.v, scale=self.inp.scale, lam=lam, causal=True, o=self.o,
                               lse=self.lse, skip_mask=False, skip_count=self.count, stream=stream)

    def work(self, skipped):
        kept = self.visited - skipped
        return FLOP_PER_PAIR * (self.visited + kept)

    def rate(self, work, ms):
        return work / (ms * 1e-3) / 1e12

    def host_bytes(self):
        return (self.inp.q.nbytes + self.inp.k.nbytes + self.inp.v.nbytes,
                self.inp.q.nbytes + self.lse.numel() * 4)

    def e2e_call(self, lam, hq, hk, hv, ho, hl):
        self.q.copy_(hq, non_blocking=True)
        self.k.copy_(hk, non_blocking=True)
        self.v.copy_(hv, non_blocking=True)
        self.call(lam)
        ho.copy_(self.o, non_blocking=True)
        hl.copy_(self.lse, non_blocking=True)


class Backward(Prefill):
    """Fixed-mask backward on the prefill workload's shape: the forward at a given
    lambda supplies o, lse and the skip mask (untimed: it runs in the warm-up call
    whenever lambda or the skip counter changes); the timed call is the backward
    alone (prep, main kernel, dq finalize).  Work: the five 128x128x128 products
    of every kept pair (S, dP, dQ, dV, dK)."""
    kind = "backward"
    e2e_in = None  # its own end-to-end step (inputs include the forward's o, lse and mask)

    def __init__(self, cfg, device, fwd=None):
        import torch

        if fwd is not None:  # share the forward workload's inputs
            self.__dict__.update({k: v for k, v in fwd.__dict__.items() if k not in ("o", "lse")})
        else:
            super().__init__(cfg, device)
        self.cfg = dict(self.cfg, workload=workload_name("backward", self.cfg))
        import synth

        c = self.cfg
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty(self.q.shape[:3], dtype=torch.float32, device=device)
        self.dout = to_dev(synth.upstream_grad(c["B"], c["Hq"], c["L"], c["d"], seed=c["seed"]), device)
        self.dq, self.dk, self.dv = torch.empty_like(self.q), torch.empty_like(self.k), torch.empty_like(self.v)
        self.ws = torch.empty(self.bl.backward_workspace_bytes(c["B"], c["Hq"], c["L"]), dtype=torch.uint8,
                              device=device)
        nq = (c["L"] + 127) // 128
        self.mask = torch.zeros((c["B"] * c["Hq"] * nq, self.bl.mask_words(nq)), dtype=torch.int32, device=device)
        self._fwd_key = None
        self.launches = 3

    def forward(self, lam):
        self.bl.prefill(self.q, self.k, self.v, scale=self.inp.scale, lam=lam, causal=True, o=self.o, lse=self.lse,
                        skip_mask=self.mask, skip_count=self.count)
        self._fwd_key = (lam, id(self.count))

    def call(self, lam, stream=None):
        if self._fwd_key != (lam, id(self.count)):
            self.forward(lam)
        return self.bl.prefill_backward(self.q, self.k, self.v, self.o, self.lse, self.dout, scale=self.inp.scale,
                                        causal=True, skip_mask=self.mask, dq=self.dq, dk=self.dk, dv=self.dv,
                                        workspace=self.ws, stream=stream)

    def work(self, skipped):
        return 5 * FLOP_PER_PAIR * (self.visited - skipped)

    def host_bytes(self):
        return (self.inp.q.nbytes * 3 + self.inp.k.nbytes + self.inp.v.nbytes + self.lse.numel() * 4 +
                self.mask.numel() * 4, self.inp.q.nbytes + self.inp.k.nbytes * 2)

    def e2e_call(self, lam, hq, hk, hv, ho, hl):
        """Every input from pinned host memory (q, k, v and the forward's o, lse, mask, plus dout),
        the backward through the public API, dq, dk, dv back to the host."""
        import torch

        if getattr(self, "_host", None) is None or self._host[0] != lam:
            self.count = torch.zeros(1, dtype=torch.int64, device=self.device)
            self.forward(lam)
            pin = lambda t: t.cpu().pin_memory()  # noqa: E731
            self._host = (lam, pin(self.o), pin(self.lse), pin(self.mask), pin(self.dout),
                          torch.empty(self.q.shape, dtype=torch.bfloat16).pin_memory(),
                          torch.empty(self.k.shape, dtype=torch.bfloat16).pin_memory(),
                          torch.empty(self.v.shape, dtype=torch.bfloat16).pin_memory())
        _, h_o, h_lse, h_mask, h_do, h_dq, h_dk, h_dv = self._host
        for dst, src in ((self.q, hq), (self.k, hk), (self.v, hv), (self.o, h_o), (self.lse, h_lse),
                         (self.mask, h_mask), (self.dout, h_do)):
            dst.copy_(src, non_blocking=True)
        self.bl.prefill_backward(self.q, self.k, self.v, self.o, self.lse, self.dout, scale=self.inp.scale,
                                 causal=True, skip_mask=self.mask, dq=self.dq, dk=self.dk, dv=self.dv,
                                 workspace=self.ws)
        h_dq.copy_(self.dq, non_blocking=True)
        h_dk.copy_(self.dk, non_blocking=True)
        h_dv.copy_(self.dv, non_blocking=True)


class Decode:
    kind = "decode"
    unit = "GB/s"
    bound = "hbm"
    seed_splits = False
    e2e_in = ("q", "k", "v")
    e2e_out = ("o", "lse")
    e2e_private = ("ws",)

    def __init__(self, cfg, device):
        import synth

        self.cfg = cfg
        self.device = device
        c = cfg
        self.inp = synth.planted_decode(c["B"], c["Hq"], c["Hkv"], c["Lk"], c["d"], seed=c["seed"], reading="blk")
        self.q, self.k, self.v = (to_dev(x, device) for x in (self.inp.q, self.inp.k, self.inp.v))
        import torch

        import block_sparse_flashattention_tcgen05_b200 as bl

        self.bl = bl
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty(self.q.shape[:3], dtype=torch.float32, device=device)
        self.ws = torch.empty(bl.decode_workspace_bytes(c["B"], c["Hq"], 1, 128, c["splits"]), dtype=torch.uint8,
                              device=device)
        self.visited = bl.visited_pairs(c["B"], c["Hq"], c["Hkv"], 1, c["Lk"], False, True)
        self.launches = 2

    def calibrate(self):
        gaps, _, _ = self.bl.calibrate(self.q, self.k, scale=self.inp.scale, causal=False, mode="decode",
                                       num_splits=self.cfg["splits"], seed_splits=self.seed_splits)
        return gaps.cpu().numpy()

    def call(self, lam, stream=None):
        return self.bl.decode(self.q, self.k, self.v, scale=self.inp.scale, lam=lam, num_splits=self.cfg["splits"],
                              o=self.o, lse=self.lse, skip_mask=False, skip_count=self.count, workspace=self.ws,
                              stream=stream, seed_splits=self.seed_splits)

    def work(self, skipped):
        c = self.cfg
        blk_bytes = 64 * c["d"] * 2
        k_bytes = c["B"] * c["Hkv"] * c["Lk"] * c["d"] * 2
        kept = self.visited - skipped
        qo = self.inp.q.nbytes * 2 + self.lse.numel() * 4
        return k_bytes + kept * blk_bytes + qo

    def rate(self, work, ms):
        return work / (ms * 1e-3) / 1e9

    def host_bytes(self):
        return (self.inp.q.nbytes + self.inp.k.nbytes + self.inp.v.nbytes,
                self.inp.q.nbytes + self.lse.numel() * 4)

    def e2e_call(self, lam, hq, hk, hv, ho, hl):
        self.q.copy_(hq, non_blocking=True)
        self.k.copy_(hk, non_blocking=True)
        self.v.copy_(hv, non_blocking=True)
        self.call(lam)
        ho.copy_(self.o, non_blocking=True)
        hl.copy_(self.lse, non_blocking=True)


class DecodeSeeded(Decode):
    """The same decode with split seeding: splits after the first start their
    running max at block 0's row maxima.  Effective bytes are counted as for
    Decode (the extra block-0 read of each split is overhead, not work)."""

    kind = "decode_seeded"
    seed_splits = True


class DecodeFp8(Decode):
    """The batch-32 GQA decode over an FP8 (e4m3) copy of the same cache, per-tensor
    scales (max |x| / 448), quantised on the device.  Effective bytes: all K bytes
    (1 per element), kept V blocks (8 KiB each), q and o.  λ: the bf16 decode's
    calibration (the sweep reports the sparsity each λ reaches here)."""

    kind = "decode_fp8"
    e2e_in = None  # its own end-to-end step (the e4m3 cache)

    def __init__(self, src, device):
        import torch

        self.__dict__.update(src.__dict__)
        self.cfg = dict(src.cfg, workload=workload_name("decode_fp8", src.cfg))

        def quant(x):
            sc = float(x.float().abs().max().item()) / 448.0
            return (x.float() / sc).clamp(-448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8), sc

        self.k8, self.k_scale = quant(src.k)
        self.v8, self.v_scale = quant(src.v)
        self.launches = 2

    def call(self, lam, stream=None):
        return self.bl.decode_fp8(self.q, self.k8, self.v8, scale=self.inp.scale, k_scale=self.k_scale,
                                  v_scale=self.v_scale, lam=lam, num_splits=self.cfg["splits"], o=self.o,
                                  lse=self.lse, skip_mask=False, skip_count=self.count, workspace=self.ws,
                                  stream=stream)

    def work(self, skipped):
        c = self.cfg
        kept = self.visited - skipped
        qo = self.inp.q.nbytes * 2 + self.lse.numel() * 4
        return c["B"] * c["Hkv"] * c["Lk"] * c["d"] + kept * 64 * c["d"] + qo

    def host_bytes(self):
        return (self.inp.q.nbytes + self.k8.numel() + self.v8.numel(), self.inp.q.nbytes + self.lse.numel() * 4)

    def e2e_call(self, lam, hq, hk, hv, ho, hl):
        """q and the e4m3 cache from pinned host memory, o and lse back."""
        if getattr(self, "_h8", None) is None:
            self._h8 = (self.k8.cpu().pin_memory(), self.v8.cpu().pin_memory())
        self.q.copy_(hq, non_blocking=True)
        self.k8.copy_(self._h8[0], non_blocking=True)
        self.v8.copy_(self._h8[1], non_blocking=True)
        self.call(lam)
        ho.copy_(self.o, non_blocking=True)
        hl.copy_(self.lse, non_blocking=True)


class DecodeMqa(Decode):
    """Decode with a 128-row tile (128 query heads on one KV head): the tcgen05 kernel."""

    kind = "decode_mqa"


class DecodeMqaSeeded(DecodeMqa):
    """The same MQA decode with split seeding (splits after the first start their running
    max at block 0's row maxima), which lifts the cap that 16 restarted splits put on its
    sparsity.  Effective bytes as for the MQA decode (the extra block-0 reads are overhead)."""

    kind = "decode_mqa_seeded"
    seed_splits = True


class DecodePaged:
    """Decode over a paged, ragged cache: the batch-32 GQA decode's keys, each
    sequence cut to its own length (uniform in [min_len, Lk], seeded) and
    scattered into randomly ordered 64-key pages.  Effective bytes: each
    sequence's own keys, kept V blocks, q and o."""

    kind = "decode_paged"
    unit = "GB/s"
    bound = "hbm"

    def __init__(self, src, device, min_len=8192, seed=11):
        import numpy as np
        import torch

        self.bl = src.bl
        self.device = device
        c = src.cfg
        self.cfg = dict(c, workload=f"decode GQA, paged 64-key cache, lengths {min_len}..{c['Lk']}, 16 splits",
                        min_len=min_len)
        self.inp = src.inp
        B, Hkv, L, d = src.inp.k.shape
        assert L % 64 == 0, "the cache length must be whole pages"
        rng = np.random.default_rng(seed)
        self.lens = rng.integers(min_len, L + 1, size=B).astype(np.int32)
        npg = (self.lens + 63) // 64
        num_pages = int(npg.sum())
        order = rng.permutation(num_pages).astype(np.int32)
        max_pages = (L + 63) // 64
        table = np.zeros((B, max_pages), np.int32)
        kp = torch.empty((num_pages, Hkv, 64, d), dtype=torch.bfloat16, device=device)
        vp = torch.empty_like(kp)
        at = 0
        for b in range(B):
            n = int(npg[b])
            ids = order[at:at + n]
            at += n
            table[b, :n] = ids
            idx = torch.from_numpy(ids.astype(np.int64)).to(device)
            kp[idx] = src.k[b, :, : n * 64].reshape(Hkv, n, 64, d).transpose(0, 1)
            vp[idx] = src.v[b, :, : n * 64].reshape(Hkv, n, 64, d).transpose(0, 1)
        self.kp, self.vp = kp, vp
        self.table = torch.from_numpy(table).to(device)
        self.lens_dev = torch.from_numpy(self.lens).to(device)
        self.q, self.o, self.lse, self.ws = src.q, src.o, src.lse, src.ws
        self.visited = int(Hkv * npg.sum())
        self.key_bytes = int(Hkv * self.lens.sum()) * d * 2
        self.launches = 2

    def call(self, lam, stream=None):
        return self.bl.decode_paged(self.q, self.kp, self.vp, self.table, self.lens_dev, scale=self.inp.scale, lam=lam,
                                    num_splits=self.cfg["splits"], o=self.o, lse=self.lse, skip_mask=False,
                                    skip_count=self.count, workspace=self.ws, stream=stream)

    def lambdas(self):
        """lambda for each target by bisection on the measured skip count (monotone in lambda)."""
        import math

        import torch

        self.count = torch.zeros(1, dtype=torch.int64, device=self.device)

        def frac(lam):
            self.call(lam)
            torch.cuda.synchronize()
            return int(self.count.item()) / self.visited

        top = frac(1 - 1e-7)
        out = {0.0: (0.0, 0.0), "max": (1 - 1e-7, top)}
        for t in TARGETS[1:]:
            if top + 0.02 < t:
                out[t] = (1 - 1e-7, top)
                continue
            lo, hi = math.log(1e-9), math.log(1 - 1e-7)
            for _ in range(22):
                mid = 0.5 * (lo + hi)
                if frac(math.exp(mid)) < t:
                    lo = mid
                else:
                    hi = mid
            out[t] = (math.exp(hi), frac(math.exp(hi)))
        return out

    def work(self, skipped):
        kept = self.visited - skipped
        return self.key_bytes + kept * 64 * 128 * 2 + self.inp.q.nbytes * 2 + self.lse.numel() * 4

    def rate(self, work, ms):
        return work / (ms * 1e-3) / 1e9


class Mla:
    """MLA decode: 576-column latent cache (V = first 512 columns), all heads in one tile."""

    kind = "mla"
    unit = "GB/s"
    bound = "hbm"
    e2e_in = ("q", "k")  # v is the same tensor as k
    e2e_out = ("o", "lse")
    e2e_private = ("ws",)

    def __init__(self, cfg, device):
        import synth

        self.cfg = cfg
        self.device = device
        c = cfg
        self.inp = synth.planted_mla(c["B"], c["Hq"], c["Lk"], seed=c["seed"], reading="blk")
        self.q, self.k = (to_dev(x, device) for x in (self.inp.q, self.inp.k))
        self.v = self.k
        import torch

        import block_sparse_flashattention_tcgen05_b200 as bl

        self.bl = bl
        self.o = torch.empty((c["B"], c["Hq"], 1, 512), dtype=torch.bfloat16, device=device)
        self.lse = torch.empty((c["B"], c["Hq"], 1), dtype=torch.float32, device=device)
        self.ws = torch.empty(bl.decode_workspace_bytes(c["B"], c["Hq"], 1, 512, c["splits"]), dtype=torch.uint8,
                              device=device)
        self.visited = bl.visited_pairs(c["B"], c["Hq"], 1, 1, c["Lk"], False, True)
        self.launches = 2

    def calibrate(self):
        gaps, _, _ = self.bl.calibrate(self.q, self.k, scale=self.inp.scale, causal=False, mode="decode",
                                       num_splits=self.cfg["splits"], dv=512,
                                       seed_splits=self.cfg.get("seed_splits", False))
        return gaps.cpu().numpy()

    def call(self, lam, stream=None):
        return self.bl.decode(self.q, self.k, self.k, scale=self.inp.scale, lam=lam, num_splits=self.cfg["splits"],
                              dv=512, o=self.o, lse=self.lse, skip_mask=False, skip_count=self.count,
                              workspace=self.ws, stream=stream, seed_splits=self.cfg.get("seed_splits", False))

    def work(self, skipped):
        c = self.cfg
        return c["B"] * c["Lk"] * 576 * 2 + self.inp.q.nbytes + self.o.numel() * 2 + self.lse.numel() * 4

    def flops(self, skipped):
        c = self.cfg
        kept = self.visited - skipped
        return 2 * c["Hq"] * 64 * 576 * self.visited + 2 * c["Hq"] * 64 * 512 * kept

    def host_bytes(self):
        return self.inp.q.nbytes + self.inp.k.nbytes, self.o.numel() * 2 + self.lse.numel() * 4

    def e2e_call(self, lam, hq, hk, hv, ho, hl):
        self.q.copy_(hq, non_blocking=True)
        self.k.copy_(hk, non_blocking=True)
        self.call(lam)
        ho.copy_(self.o, non_blocking=True)
        hl.copy_(self.lse, non_blocking=True)

    def rate(self, work, ms):
        return work / (ms * 1e-3) / 1e9


def r4(x):
    """Four significant digits (the JSON line stays short enough to be read whole)."""
    return None if x is None else float(f"{x:.4g}")


def per_head_sparsity(wl, lam):
    """Skipped / visited pairs of each head at lambda (one extra call with the skip
    mask, outside any timed region): (min, median, max) over the heads.  Prefill:
    each query head (its tiles' pairs); decode: each KV head, over the batch (the
    tile of a decode is a KV head's group)."""
    import numpy as np
    import torch

    c = wl.cfg
    wl.count = torch.zeros(1, dtype=torch.int64, device=wl.device)
    if wl.kind in ("prefill", "backward"):
        nq = (c["L"] + 127) // 128
        nb = (c["L"] + 127) // 128
        _, _, m, _ = wl.bl.prefill(wl.q, wl.k, wl.v, scale=wl.inp.scale, lam=lam, causal=True, o=wl.o,
                                   lse=wl.lse, skip_mask=True, skip_count=wl.count)
        heads, rows_per_head = c["B"] * c["Hq"], nq
        vis = np.full(c["Hq"], wl.visited / heads)
    else:
        nb = (c["Lk"] + 63) // 64
        _, _, m, _ = wl.bl.decode(wl.q, wl.k, wl.v, scale=wl.inp.scale, lam=lam, num_splits=c["splits"], o=wl.o,
                                  lse=wl.lse, skip_mask=True, skip_count=wl.count, workspace=wl.ws,
                                  seed_splits=getattr(wl, "seed_splits", False))
        heads, rows_per_head = c["Hkv"], 1
        vis = np.full(c["Hkv"], float(c["B"] * nb))
    torch.cuda.synchronize()
    w = m.cpu().numpy().astype(np.uint32)
    ones = np.zeros(w.shape[0], np.int64)
    for bit in range(32):
        ones += ((w >> np.uint32(bit)) & np.uint32(1)).astype(np.int64).sum(axis=1)
    if wl.kind in ("prefill", "backward"):
        per = ones.reshape(c["B"], c["Hq"], rows_per_head).sum(axis=(0, 2)) / vis
    else:
        per = ones.reshape(c["B"], c["Hkv"]).sum(axis=0) / vis
    return [r4(float(per.min())), r4(float(np.median(per))), r4(float(per.max()))]


def decision_overhead(wl, flush, rounds=4, per_round=3):
    """The prefill against its measurement instance with the skip decision compiled
    out, both at lambda = 0 (the same dense result), timed in interleaved rounds:
    (median ms of each, speed of the real kernel relative to the no-vote one)."""
    import torch

    stream = torch.cuda.current_stream()
    t = {"vote": [], "novote": []}
    fns = {"vote": wl.bl.prefill, "novote": wl.bl.measure_prefill_novote}
    for name, fn in fns.items():  # warm-up
        for _ in range(2):
            fn(wl.q, wl.k, wl.v, scale=wl.inp.scale, lam=0.0, causal=True, o=wl.o, lse=wl.lse, skip_mask=False,
               skip_count=False)
    for _ in range(rounds):
        for name, fn in fns.items():
            for _ in range(per_round):
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                flush.zero_()
                a.record(stream)
                fn(wl.q, wl.k, wl.v, scale=wl.inp.scale, lam=0.0, causal=True, o=wl.o, lse=wl.lse,
                   skip_mask=False, skip_count=False)
                b.record(stream)
                torch.cuda.synchronize()
                t[name].append(a.elapsed_time(b))
    mv, mn = statistics.median(t["vote"]), statistics.median(t["novote"])
    return {"ms": r4(mv), "ms_no_vote": r4(mn), "speed_vs_no_vote": r4(mn / mv), "pages": "0.96-1.00"}


def lambdas_for_targets(wl, gaps):
    out = {}
    for t in TARGETS:
        if t == 0.0:
            out[t] = (0.0, 0.0)
            continue
        lam, ach = wl.bl.calibrate_threshold(gaps, t)
        if ach + 0.02 < t:  # unreachable target: the highest reachable sparsity
            lam, ach = wl.bl.calibrate_threshold(gaps, 1.0)
        out[t] = (lam, ach)
    out["max"] = wl.bl.calibrate_threshold(gaps, 1.0)  # (lambda, sparsity) as lambda -> 1
    return out


def timed_launches(wl, lam, steps, warmup, flush, sampler=None):
    """Per-launch device times (ms) with CUDA events on the launching stream, L2 flushed before each."""
    import torch

    stream = torch.cuda.current_stream()
    wl.count = torch.zeros(1, dtype=torch.int64, device=wl.device)
    for _ in range(warmup):
        wl.call(lam)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    t0 = time.time()
    for i in range(steps):
        flush.zero_()
        ev[i][0].record(stream)
        wl.call(lam)
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    t1 = time.time()
    if sampler:
        sampler.mark(t0, t1)
    ms = [a.elapsed_time(b) for a, b in ev]
    skipped = int(wl.count.item())
    return ms, skipped


def e2e_measure(wl, lam, steps, warmup):
    """The metric end to end through the public API, from and to pinned host memory.

    Every step copies its inputs host -> device, makes the call and copies its result
    device -> host, all inside the timed region.  Where the workload names its device
    tensors (e2e_in / e2e_out), steps run as a pipeline over two sets of device buffers
    and three streams: step i's host -> device copy overlaps step i-1's call and step
    i-2's device -> host copy (PCIe carries both directions at once).  Otherwise the
    workload's own step runs serially on one stream."""
    import copy

    import torch

    if getattr(wl, "e2e_in", None) is None:
        return _e2e_serial(wl, lam, steps, warmup)
    wl.count = torch.zeros(1, dtype=torch.int64, device=wl.device)
    sets = [wl, copy.copy(wl)]
    for name in wl.e2e_in + wl.e2e_out + wl.e2e_private + ("count",):
        setattr(sets[1], name, getattr(wl, name).clone())
    if isinstance(wl, Mla):
        sets[1].v = sets[1].k
    host_in = {name: getattr(wl, name).cpu().pin_memory() for name in wl.e2e_in}
    host_out = [{name: torch.empty(getattr(wl, name).shape, dtype=getattr(wl, name).dtype).pin_memory()
                 for name in wl.e2e_out} for _ in sets]
    s_h2d, s_call, s_d2h = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev = {k: [torch.cuda.Event() for _ in sets] for k in ("h2d", "call", "d2h")}
    used = [False, False]

    def step(i):
        k = i % 2
        w = sets[k]
        with torch.cuda.stream(s_h2d):
            if used[k]:
                s_h2d.wait_event(ev["call"][k])  # the previous call on this set has read its inputs
            for name in w.e2e_in:
                getattr(w, name).copy_(host_in[name], non_blocking=True)
            ev["h2d"][k].record(s_h2d)
        s_call.wait_event(ev["h2d"][k])
        if used[k]:
            s_call.wait_event(ev["d2h"][k])  # the previous result of this set has left the device
        w.call(lam, stream=s_call)
        ev["call"][k].record(s_call)
        with torch.cuda.stream(s_d2h):
            s_d2h.wait_event(ev["call"][k])
            for name in w.e2e_out:
                host_out[k][name].copy_(getattr(w, name), non_blocking=True)
            ev["d2h"][k].record(s_d2h)
        used[k] = True

    for i in range(max(2, warmup)):
        step(i)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(s_h2d)
    s_call.wait_event(a)
    s_d2h.wait_event(a)
    for i in range(steps):
        step(i)
    s_d2h.wait_event(ev["call"][(steps - 1) % 2])
    b.record(s_d2h)  # after every copy out, which follows every call and copy in
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    skipped = int(wl.count.item())
    hb, db = wl.host_bytes()
    return ms, skipped, hb, db


def _e2e_serial(wl, lam, steps, warmup):
    import torch

    hq, hk = to_pinned(wl.inp.q), to_pinned(wl.inp.k)
    hv = to_pinned(wl.inp.v) if wl.inp.v is not None else None  # MLA: V is the K buffer
    ho = torch.empty(wl.o.shape, dtype=torch.bfloat16).pin_memory()
    hl = torch.empty(wl.lse.shape, dtype=torch.float32).pin_memory()
    wl.count = torch.zeros(1, dtype=torch.int64, device=wl.device)
    for _ in range(max(1, warmup)):
        wl.e2e_call(lam, hq, hk, hv, ho, hl)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        wl.e2e_call(lam, hq, hk, hv, ho, hl)
    b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    skipped = int(wl.count.item())
    hb, db = wl.host_bytes()
    return ms, skipped, hb, db


# ------------------------------------------------------------- calibration sweep
def calibration_sweep(device, lengths, targets=(0.3, 0.4, 0.5, 0.6, 0.7, 0.8), B=1, Hq=32, Hkv=8, seed=7):
    """Fit lambda*L = alpha*exp(beta*s) across context lengths (one decision-only pass per L).

    For each L: gaps from blasst_calibrate; per target s the lambda reaching s (gap quantile), a = lambda*L.
    Fit over all reachable (L, s) points with blasst_calibrate_fit, then report, per L and s, the sparsity
    reached by the fitted lambda = a(s)/L, and by one fixed lambda (the one giving 50% at the middle L)."""
    import numpy as np
    import torch

    import block_sparse_flashattention_tcgen05_b200 as bl
    import synth

    per_L = {}
    pts_L, pts_lam, pts_s = [], [], []
    for L in lengths:
        inp = synth.planted_prefill(B, Hq, Hkv, L, 128, seed=seed, reading="blk")
        q, k = to_dev(inp.q, device), to_dev(inp.k, device)
        t0 = time.time()
        gaps, _, _ = bl.calibrate(q, k, scale=inp.scale, causal=True, mode="prefill")
        torch.cuda.synchronize()
        g = gaps.cpu().numpy()
        per_L[L] = dict(gaps=g, visited=int(np.count_nonzero(~np.isnan(g))), calib_s=time.time() - t0)
        for t in targets:
            lam, ach = bl.calibrate_threshold(g, t)
            if lam > 0 and abs(ach - t) < 0.01:
                pts_L.append(L)
                pts_lam.append(lam)
                pts_s.append(ach)
        del q, k, gaps
    alpha, beta = bl.calibrate_fit(pts_L, pts_lam, pts_s)

    def sparsity_at(g, lam):
        fin = g[~np.isnan(g)]
        return float(np.count_nonzero(fin < math.log(lam))) / fin.size if lam > 0 else 0.0

    mid = lengths[len(lengths) // 2]
    lam_fixed, _ = bl.calibrate_threshold(per_L[mid]["gaps"], 0.5)
    rows = []
    errs = []
    for L in lengths:
        g = per_L[L]["gaps"]
        for t in targets:
            lam_fit = min(alpha * math.exp(beta * t) / L, 1.0 - 1e-7)
            sp = sparsity_at(g, lam_fit)
            errs.append(abs(sp - t))
            rows.append({"L": L, "target": t, "a_fit": alpha * math.exp(beta * t), "lambda_fit": lam_fit,
                         "achieved": sp, "abs_error": abs(sp - t)})
    fixed = {str(L): sparsity_at(per_L[L]["gaps"], lam_fixed) for L in lengths}
    cal50 = {str(L): sparsity_at(per_L[L]["gaps"], min(alpha * math.exp(beta * 0.5) / L, 1 - 1e-7))
             for L in lengths}
    return {"alpha": alpha, "beta": beta, "points": len(pts_s), "mean_abs_sparsity_error": float(np.mean(errs)),
            "max_abs_sparsity_error": float(np.max(errs)), "per_point": rows,
            "fixed_lambda": {"lambda": lam_fixed, "sparsity_by_L": fixed},
            "calibrated_50pct_sparsity_by_L": cal50,
            "workload": f"prefill GQA B={B} Hq={Hq} Hkv={Hkv} d=128 causal, 'blk' inputs seed {seed}"}


# ------------------------------------------------------------------ CPU baseline
def oracle_sample(wl_kind, cfg, lam_target=0.75, budget_s=10.0, seed_tiles=0):
    """Time the fp64 oracle (as it stands) on a bounded sample of query tiles.

    Returns dict(value, unit, cores, kind, sample)."""
    import numpy as np

    import oracle
    import synth

    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    rng = np.random.default_rng(seed_tiles)
    if wl_kind == "backward":
        return oracle_backward_sample(cfg, lam_target, budget_s, seed_tiles)
    if wl_kind == "prefill":
        c = cfg
        inp = synth.planted_prefill(c["B"], c["Hq"], c["Hkv"], c["L"], c["d"], seed=c["seed"], reading="blk")
        nq = c["L"] // 128
        n_tiles = c["B"] * c["Hq"] * nq
        # tiles from the last quarter of the sequence (long rows); count grows until the budget is used
        cand = [t for t in range(n_tiles) if (t % nq) >= nq * 3 // 4]
        rng.shuffle(cand)
        kw = dict(scale=inp.scale, causal=True)
        units = lambda r: FLOP_PER_PAIR * (r["n_visited"] * 2 - r["n_skipped"]) / 1e12  # noqa: E731
        unit = "TFLOP/s"
    elif wl_kind == "mla":
        c = cfg
        # per-sequence work is the same at any batch: 4 sequences keep the generator cheap
        inp = synth.planted_mla(min(4, c["B"]), c["Hq"], c["Lk"], seed=c["seed"], reading="blk")
        cand = list(range(inp.q.shape[0]))
        rng.shuffle(cand)
        kw = dict(scale=inp.scale, causal=False, is_decode=True, num_splits=c["splits"], BN=64, dv=512,
                  v_row_stride=576, seed_splits=c.get("seed_splits", False))
        n_tiles = c["B"]

        def units(r):
            return r["_tiles"] * c["Lk"] * 576 * 2 / 1e9
        unit = "GB/s"
    else:
        c = cfg
        inp = synth.planted_decode(c["B"], c["Hq"], c["Hkv"], c["Lk"], c["d"], seed=c["seed"], reading="blk")
        cand = list(range(c["B"] * c["Hkv"]))
        rng.shuffle(cand)
        kw = dict(scale=inp.scale, causal=False, is_decode=True, num_splits=c["splits"],
                  seed_splits=c.get("seed_splits", False))
        blk = 64 * c["d"] * 2
        keyb = c["Lk"] * c["d"] * 2
        n_tiles = len(cand)

        def units(r):
            return (r["_tiles"] * keyb + (r["n_visited"] - r["n_skipped"]) * blk) / 1e9
        unit = "GB/s"
    # calibrate lambda on the first tiles (their own gaps), then time
    n = max(1, min(len(cand), cores))
    t0 = time.time()
    v = inp.k if inp.v is None else inp.v
    r0 = oracle.attention(inp.q, inp.k, v, lam=0.0, tiles=cand[:n], **kw)
    dt = time.time() - t0
    lam, _ = oracle.threshold_for_sparsity(r0["gaps"][cand[:n]], r0["visited"][cand[:n]], lam_target)
    n = int(max(1, min(len(cand), n * budget_s / max(dt, 1e-3))))
    tiles = cand[:n]
    t0 = time.time()
    r = oracle.attention(inp.q, inp.k, v, lam=lam, tiles=tiles, **kw)
    dt = time.time() - t0
    r["_tiles"] = len(tiles)
    return dict(value=units(r) / dt, unit=unit, cores=cores, kind="oracle",
                sample=f"{len(tiles)} of {n_tiles} query tiles "
                       f"({'last quarter of the sequence' if wl_kind == 'prefill' else 'whole KV heads'}), "
                       f"lambda={lam:.4g} for ~{lam_target:.0%} sparsity on the sample, {dt:.1f} s",
                seconds=dt)


def oracle_backward_sample(cfg, lam_target=0.75, budget_s=10.0, seed=0):
    """Time the fp64 backward oracle (as it stands) on a bounded sample of the
    backward workload: the first Ls tokens of one KV head's query-head group
    (the oracle forms the whole Ls x Ls score matrix), its forward mask from the
    C oracle at a lambda for ~lam_target sparsity.  Ls doubles until the budget."""
    import numpy as np

    import oracle
    import synth

    c = cfg
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    G = c["Hq"] // c["Hkv"]
    kv = seed % c["Hkv"]
    inp = synth.planted_prefill(1, c["Hq"], c["Hkv"], min(c["L"], 8192), c["d"], seed=c["seed"], reading="blk")
    do = synth.upstream_grad(1, c["Hq"], min(c["L"], 8192), c["d"], seed=c["seed"])
    Ls, dt, res = 1024, 0.0, None
    while True:
        q = np.ascontiguousarray(inp.q[:, kv * G:(kv + 1) * G, :Ls])
        k = np.ascontiguousarray(inp.k[:, kv:kv + 1, :Ls])
        v = np.ascontiguousarray(inp.v[:, kv:kv + 1, :Ls])
        d_o = np.ascontiguousarray(do[:, kv * G:(kv + 1) * G, :Ls])
        f0 = oracle.attention(q, k, v, scale=inp.scale, lam=0.0, causal=True)
        lam, _ = oracle.threshold_for_sparsity(f0["gaps"], f0["visited"], lam_target)
        f = oracle.attention(q, k, v, scale=inp.scale, lam=lam, causal=True)
        t0 = time.time()
        oracle.attention_backward(q, k, v, d_o, scale=inp.scale, causal=True, skip=f["skip"])
        dt = time.time() - t0
        res = (Ls, lam, f["n_visited"] - f["n_skipped"], f["n_skipped"] / max(1, f["n_visited"]))
        if dt * 4.5 > budget_s or Ls * 2 > min(c["L"], 8192):
            break
        Ls *= 2
    Ls, lam, kept, sp = res
    return dict(value=5 * FLOP_PER_PAIR * kept / dt / 1e12, unit="TFLOP/s", cores=cores, kind="oracle",
                sample=f"first {Ls} tokens of KV head {kv}'s {G} query heads, lambda={lam:.4g} "
                       f"({sp:.0%} of pairs skipped), {dt:.1f} s", seconds=dt)


def oracle_mha1024(lam_a=32.0, budget_s=3.0):
    """The oracle on the whole 1024-token MHA prefill (planted generator,
    lambda = a/L), repeated for about budget_s; effective TFLOP/s."""
    import oracle
    import synth

    L = 1024
    inp = synth.planted_prefill(1, 1, 1, L, 128, seed=1, reading="lit", boost=False)
    n, t0 = 0, time.time()
    while True:
        r = oracle.attention(inp.q, inp.k, inp.v, scale=inp.scale, lam=lam_a / L, causal=True)
        n += 1
        if time.time() - t0 >= budget_s:
            break
    dt = time.time() - t0
    work = FLOP_PER_PAIR * (2 * r["n_visited"] - r["n_skipped"]) * n / 1e12
    return {"value": work / dt, "unit": "TFLOP/s", "sample": f"whole 1024-token MHA prefill, lambda={lam_a:g}/L, "
            f"{n} runs in {dt:.1f} s"}


def single_core_oracle(dcfg):
    """The oracle on one host core (child process, OMP_NUM_THREADS=1): the
    1024-token MHA prefill in full and a sample of the GQA decode workload."""
    import subprocess

    env = dict(os.environ, OMP_NUM_THREADS="1")
    cmd = [sys.executable, os.path.abspath(__file__), "--single-core-oracle", json.dumps(dcfg)]
    try:
        out = subprocess.run(cmd, env=env, capture_output=True, text=True, timeout=120, check=True).stdout
        return json.loads(out.strip().splitlines()[-1])
    except Exception as e:  # reported, never fatal to the GPU measurement
        return {"error": f"{type(e).__name__}: {e}"[:200]}


def _single_core_main(dcfg_json):
    dcfg = json.loads(dcfg_json)
    res = {"threads": int(os.environ.get("OMP_NUM_THREADS", "0")), "mha_prefill_1024": oracle_mha1024()}
    d = oracle_sample("decode", dcfg, budget_s=4.0)
    res["decode"] = {k: d[k] for k in ("value", "unit", "sample")}
    print(json.dumps(res), flush=True)


# -------------------------------------------------------------------------- main
def dist_setup(args):
    import torch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def aggregate(units_local, seconds_local, world):
    """Whole-job throughput: units over all ranks / max over ranks of the time."""
    if world > 1:
        import torch
        import torch.distributed as dist

        dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
        t = torch.tensor([seconds_local], dtype=torch.float64, device=dev)
        u = torch.tensor([units_local], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        dist.all_reduce(u, op=dist.ReduceOp.SUM)
        return u.item() / t.item(), t.item()
    return units_local / seconds_local, seconds_local


def run_reference(args, world, rank):
    if rank != 0:
        return
    wl_kind = args.workload
    if wl_kind == "decode_mqa":
        cfg = mqa_cfg(args.size, SIZES[args.size][1])
    else:
        cfg = SIZES[args.size][{"prefill": 0, "decode": 1, "mla": 2, "backward": 0, "decode_fp8": 1}[wl_kind]]
    cfg = dict(cfg, workload=workload_name(wl_kind, cfg))
    per_step = []
    vals = []
    budget = float(os.environ.get("BLASST_REF_STEP_SECONDS", "8"))
    for i in range(args.warmup + args.steps):
        r = oracle_sample(wl_kind, cfg, budget_s=budget, seed_tiles=i)
        if i >= args.warmup:
            per_step.append(r["seconds"])
            vals.append(r["value"])
    value = statistics.mean(vals)
    unit = r["unit"]
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": unit, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * statistics.mean(per_step),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": cfg["workload"], "lambda_target": 0.75, "reading": "blk"},
        "cpu_baseline": {"value": value, "unit": unit, "cores": r["cores"], "kind": "oracle", "sample": r["sample"]},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    if len(sys.argv) == 3 and sys.argv[1] == "--single-core-oracle":
        _single_core_main(sys.argv[2])
        return
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["mine", "reference"], default="mine")
    ap.add_argument("--workload", choices=["prefill", "decode", "mla", "backward", "decode_fp8", "decode_mqa"],
                    default="prefill")
    ap.add_argument("--size", choices=sorted(SIZES), default="full",
                    help="full = the benchmark shapes; medium = profiling size; quick = smoke-testing the bench")
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-mla", action="store_true")
    ap.add_argument("--no-64k", action="store_true")
    ap.add_argument("--no-seeded", action="store_true", help="skip the split-seeded decode rows of the sweep")
    ap.add_argument("--no-paged", action="store_true", help="skip the paged, ragged decode rows of the sweep")
    ap.add_argument("--no-mqa", action="store_true", help="skip the 128-head MQA decode rows of the sweep")
    ap.add_argument("--no-backward", action="store_true", help="skip the fixed-mask backward rows of the sweep")
    ap.add_argument("--no-fp8", action="store_true", help="skip the FP8-cache decode rows of the sweep")
    ap.add_argument("--no-calibration", action="store_true",
                    help="skip the fit of lambda*L = alpha*exp(beta*s) over L in {8K,16K,32K,64K}")
    ap.add_argument("--no-decision-overhead", action="store_true",
                    help="skip timing the prefill against its no-vote instance at lambda = 0")
    ap.add_argument("--detail-out", default=None,
                    help="also write every sweep point in full (lambda, a = lambda*L, ...) to this JSON file")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    world, rank, local = dist_setup(args)
    if args.impl == "reference":
        run_reference(args, world, rank)
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()
        return

    import torch

    import block_sparse_flashattention_tcgen05_b200 as bl

    dev = torch.device("cuda", local)
    peaks, peak_src = load_peaks()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    notes = []

    pcfg, dcfg, mcfg = SIZES[args.size]
    headline_kind = args.workload
    wls = {}
    if headline_kind == "prefill":
        try:
            wls["prefill"] = Prefill(pcfg, dev)
            wls["prefill"].count = torch.zeros(1, dtype=torch.int64, device=dev)
            wls["prefill"].call(0.0)
            torch.cuda.synchronize()
        except bl.BlasstError as e:
            if e.status != 2:
                raise
            wls.pop("prefill", None)
            notes.append("prefill kernel not available in this build; headline falls back to decode")
            headline_kind = "decode"
    if headline_kind in ("decode", "decode_fp8"):
        wls["decode"] = Decode(dcfg, dev)
    if headline_kind == "decode_fp8":
        wls["decode_fp8"] = DecodeFp8(wls["decode"], dev)
    if headline_kind == "mla":
        wls["mla"] = Mla(mcfg, dev)
    if headline_kind == "decode_mqa":
        wls["decode_mqa"] = DecodeMqa(mqa_cfg(args.size, dcfg), dev)
    if headline_kind == "backward":
        wls["backward"] = Backward(pcfg, dev)
        wls["backward"].count = torch.zeros(1, dtype=torch.int64, device=dev)
    # the headline workload is calibrated and timed before any other workload runs
    lams = {headline_kind: lambdas_for_targets(wls[headline_kind], wls[headline_kind].calibrate())}

    # ---- headline: the ~75% point of the headline workload
    wl = wls[headline_kind]
    lam75, ach75 = lams[headline_kind][0.75]
    sampler = ClockSampler(local)
    sampler.start()
    if world > 1:
        import torch.distributed as dist

        dist.barrier()
    torch.cuda.synchronize()
    ms, skipped = timed_launches(wl, lam75, args.steps, args.warmup, flush, sampler)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    work = wl.work(skipped)
    ms_mean = statistics.mean(ms)
    value, t_max = aggregate(work * args.steps, sum(ms) * 1e-3, world)
    value = value / (1e12 if wl.unit == "TFLOP/s" else 1e9)
    achieved = wl.rate(work, ms_mean)
    if wl.bound == "tensor":
        peak = peaks["bf16_tflops"]
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                "peak_source": f"{peak_src} bf16 burst"}
    else:
        peak = peaks["hbm_gbs"]
        roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                "peak_source": f"{peak_src} copy bandwidth"}

    prof = load_profile_counters(wl.kind)
    roof["traffic"] = prof.get("dram_bytes_per_launch")
    if wl.bound == "tensor":
        roof["tensor_pipe_active_pct_ncu"] = prof.get("tensor_pipe_active_pct")
    if prof:
        roof["ncu_source"] = prof.get("source")

    # ---- sweep: 0/50/75% on every workload, speedup over lambda = 0
    sweep, sweep_full = {}, {}
    if not args.no_sweep:
        if "prefill" not in wls:
            try:
                wls["prefill"] = Prefill(pcfg, dev)
            except bl.BlasstError as e:
                if e.status != 2:
                    raise
        if "decode" not in wls:
            wls["decode"] = Decode(dcfg, dev)
        if not args.no_seeded:
            ws = DecodeSeeded.__new__(DecodeSeeded)  # shares the decode workload's inputs and buffers
            ws.__dict__.update(wls["decode"].__dict__)
            wls["decode_seeded"] = ws
        if not args.no_fp8:
            wls["decode_fp8"] = DecodeFp8(wls["decode"], dev)
        if not args.no_paged:
            wls["decode_paged"] = DecodePaged(wls["decode"], dev,
                                              min_len=min(8192, wls["decode"].cfg["Lk"] // 4))
        if not args.no_mqa and "decode_mqa" not in wls:
            wls["decode_mqa"] = DecodeMqa(mqa_cfg(args.size, dcfg), dev)
        if not args.no_mqa and not args.no_seeded and "decode_mqa" in wls:
            wm = DecodeMqaSeeded.__new__(DecodeMqaSeeded)  # shares the MQA workload's inputs and buffers
            wm.__dict__.update(wls["decode_mqa"].__dict__)
            wls["decode_mqa_seeded"] = wm
        if "mla" not in wls and not args.no_mla:
            wls["mla"] = Mla(mcfg, dev)
        if "prefill" in wls and "backward" not in wls and not args.no_backward:
            wls["backward"] = Backward(pcfg, dev, fwd=wls["prefill"])
        if args.size == "full" and "prefill" in wls and not args.no_64k:
            wls["prefill_64k"] = Prefill(PREFILL_64K, dev)
        if "backward" in wls and "prefill" in lams and "backward" not in lams:
            lams["backward"] = lams["prefill"]  # same inputs, same forward masks
        if "decode_fp8" in wls and "decode" in lams and "decode_fp8" not in lams:
            lams["decode_fp8"] = lams["decode"]
        for k, w in wls.items():
            if k not in lams:
                lams[k] = w.lambdas() if hasattr(w, "lambdas") else lambdas_for_targets(w, w.calibrate())
        rounds = 4
        for kind, w in wls.items():
            # the sparsity points of a workload are timed round-robin, so that a drift of
            # clocks or temperature during the sweep lands on all of them alike; odd rounds
            # take the points in reverse order, so that no point always follows the dense one
            # (whose power draw lowers the clock of what runs right after it)
            times = {t: [] for t in TARGETS}
            sk_by_t = {}
            for rnd in range(rounds):
                for t in (TARGETS if rnd % 2 == 0 else TARGETS[::-1]):
                    ms_t, sk_by_t[t] = timed_launches(w, lams[kind][t][0], max(2, args.steps // (2 * rounds)),
                                                      3 if rnd == 0 else 1, flush)
                    times[t] += ms_t
            base = statistics.median(times[0.0])
            pk = peaks["bf16_tflops"] if w.bound == "tensor" else peaks["hbm_gbs"]
            spk = SPEC_PEAKS["bf16_tflops"] if w.bound == "tensor" else SPEC_PEAKS["hbm_gbs"]
            pts, full = [], {}
            for t in TARGETS:
                lam = lams[kind][t][0]
                sk = sk_by_t[t]
                med = statistics.median(times[t])
                r = w.rate(w.work(sk), med)
                pt = [r4(sk / w.visited), r4(med), r4(r), r4(r / pk), r4(r / spk), r4(base / med)]
                row = {"lambda": lam, "a=lambda*L": lam * (w.cfg.get("L") or w.cfg.get("Lk")),
                       "sparsity": sk / w.visited, "ms": med, "value": r, "unit": w.unit,
                       "frac_of_measured_peak": r / pk, "frac_of_spec_peak": r / spk, "speedup_vs_lambda0": base / med}
                if hasattr(w, "flops"):  # MLA: the tensor side too
                    tf = w.flops(sk) / (med * 1e-3) / 1e12
                    pt.append(r4(tf / peaks["bf16_tflops"]))
                    row.update(tflops=tf, tensor_frac_of_measured_peak=tf / peaks["bf16_tflops"])
                pts.append(pt)
                full[f"{int(t * 100)}%"] = row
            full["max_reachable_sparsity"] = lams[kind]["max"][1]
            sweep[kind] = {"u": w.unit, "pts": pts, "max_s": r4(lams[kind]["max"][1])}
            sweep_full[kind] = full

    # ---- per-head sparsity distribution at the ~75% point (A10: report the per-head distribution)
    per_head = {}
    for kind in ("prefill", "prefill_64k", "decode"):
        if kind in wls and kind in lams:
            per_head[kind] = per_head_sparsity(wls[kind], lams[kind][0.75][0])

    # ---- the decision's cost: prefill against its no-vote instance at lambda = 0
    dec_ovh = None
    if not args.no_decision_overhead and "prefill" in wls:
        dec_ovh = decision_overhead(wls["prefill"], flush)

    # ---- calibration fit across context lengths (prefill-shaped decision pass)
    calib = calib_full = None
    if not args.no_calibration and "prefill" in wls:
        lengths = (8192, 16384, 32768, 65536) if args.size == "full" else (2048, 4096, 8192)
        calib_full = calibration_sweep(dev, lengths)
        err_by_L = {}
        for row in calib_full["per_point"]:
            err_by_L.setdefault(str(row["L"]), []).append(row["abs_error"])
        calib = {"alpha": r4(calib_full["alpha"]), "beta": r4(calib_full["beta"]), "points": calib_full["points"],
                 "mean_abs_err": r4(calib_full["mean_abs_sparsity_error"]),
                 "max_abs_err": r4(calib_full["max_abs_sparsity_error"]),
                 "mean_abs_err_by_L": {L: r4(statistics.mean(v)) for L, v in err_by_L.items()},
                 "targets": [0.3, 0.4, 0.5, 0.6, 0.7, 0.8]}

    # ---- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        e_ms, e_sk, hb, db = e2e_measure(wl, lam75, max(3, args.steps // 4), 1)
        e_val, _ = aggregate(wl.work(e_sk), e_ms * 1e-3, world)
        e2e = {"value": e_val / (1e12 if wl.unit == "TFLOP/s" else 1e9), "unit": wl.unit, "h2d_bytes_per_step": hb,
               "d2h_bytes_per_step": db, "ms_per_step": e_ms}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = oracle_sample(headline_kind, wl.cfg, budget_s=float(os.environ.get("BLASST_CPU_SECONDS", "12")))
        cpu = {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample")}
        cpu["cpu_model"] = cpu_model()
        cpu["nproc"] = os.cpu_count()
        # per-tile work is the same at any batch: a batch of 4 keeps the generator cheap
        cpu["single_core"] = single_core_oracle(dict(dcfg, B=min(4, dcfg["B"])))

    cfgd = {"workload": wl.cfg["workload"], "lambda": lam75, "target_sparsity": 0.75, "achieved_sparsity":
            skipped / wl.visited, "visited_pairs": wl.visited, "reading": "blk",
            "l2": "flushed (256 MiB write) before every timed launch"}
    for k in ("B", "Hq", "Hkv", "L", "Lk", "d", "splits"):
        if k in wl.cfg:
            cfgd[k] = wl.cfg[k]
    roof["frac_of_spec"] = roof["achieved"] / (SPEC_PEAKS["bf16_tflops"] if wl.bound == "tensor"
                                              else SPEC_PEAKS["hbm_gbs"])
    roof["spec_peak"] = SPEC_PEAKS["bf16_tflops"] if wl.bound == "tensor" else SPEC_PEAKS["hbm_gbs"]
    line = {
        "metric": METRIC, "value": value, "unit": wl.unit, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": t_max * 1e3 / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": cfgd,
        "roofline": roof, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": wl.launches * args.steps,
        "clocks": clocks, "notes": notes,
        # the keys below are kept short and last, so that a reader of the line's tail sees all of them
        "decision_overhead": dec_ovh, "per_head_sparsity_75": per_head, "calibration": calib,
        "sweep_cols": ["sparsity", "ms", "value", "frac_measured", "frac_spec", "speedup_vs_lambda0",
                       "(mla) tensor_frac_measured"],
        "sweep": sweep,
    }
    if args.detail_out and rank == 0:
        with open(args.detail_out, "w") as f:
            json.dump({"line": line, "sweep": sweep_full, "calibration": calib_full,
                       "lambdas": {k: {str(t): v for t, v in d.items()} for k, d in lams.items()}}, f, indent=1,
                      default=str)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
