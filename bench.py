#!/usr/bin/env python
"""Benchmark: effective TFLOP/s of the block-sparse attention forward on B200.

Default workload (the largest one, and the most computed work): GNA-like 3-D
video neighborhood attention, B=1 H=24 d=128, 256 text tokens + a 16x48x80
video grid (61,696 tokens), tiles 4x8x8, window 8x16x24, stride 1x1x1, so
6272 of the 7521 kept tile pairs per head are partial and take the fine mask.
One step = the whole hot path on one batch: bsa_permute_tiles (Q, K, V into
tile order) + bsa_build_mask (GNA) + bsa_forward + bsa_unpermute_tiles (O).

Effective FLOPs count only computed blocks: 4 * block_q * block_k * d per kept
(b, h, query block, KV block); partial tiles count in full; skip heads count 0.

Usage:
  python bench.py [--gpus N] [--steps K] [--warmup W] [--config c5f|c5s|c4|c3|c2|c1]
  python bench.py --impl reference ...   (the fp64 oracle on host cores)
Under torchrun every rank runs its own independent instance (weak scaling, no
data-path collective); the timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "effective TFLOP/s of block-sparse attn fwd & % of BF16 peak; speedup vs dense"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None, help="default: per workload (about 2 s of timed work)")
    ap.add_argument("--warmup", type=int, default=None)
    ap.add_argument("--impl", default="bsa", choices=["bsa", "reference"])
    ap.add_argument("--config", default="c5f", choices=["c1", "c2", "c3", "c4", "c5s", "c5f"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-fp8", action="store_true", help="skip the e4m3 forward leg (d = 128 workloads)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="oracle sample budget")
    ap.add_argument("--shard", default="replicas", choices=["replicas", "heads"],
                    help="N > 1: independent replicas per GPU (weak scaling, default), or one problem split "
                         "by heads with O all-gathered inside every step (strong scaling)")
    a = ap.parse_args()
    steps, warmup = DEFAULT_STEPS[a.config]
    a.steps = steps if a.steps is None else a.steps
    a.warmup = warmup if a.warmup is None else a.warmup
    return a


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, local_rank: int, period_s: float = 0.005):
        self.period = period_s
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self.err = None
        self._stop = threading.Event()
        self._thr = None
        try:
            import pynvml
            pynvml.nvmlInit()
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            idx = local_rank
            if vis:
                ids = [x.strip() for x in vis.split(",") if x.strip()]
                if local_rank < len(ids) and ids[local_rank].isdigit():
                    idx = int(ids[local_rank])
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # noqa: BLE001
            self.err = repr(e)
            self.nv = None

    def _run(self):
        nv = self.nv
        get_r = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = get_r(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception as e:  # noqa: BLE001
                self.err = repr(e)
            time.sleep(self.period)

    def start(self):
        if self.nv is not None:
            self._thr = threading.Thread(target=self._run, daemon=True)
            self._thr.start()

    def stop(self):
        self._stop.set()
        if self._thr is not None:
            self._thr.join()

    def summary(self):
        if self.nv is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": self.err}
        out = {"sm_mhz": statistics.median(self.samples) if self.samples else None,
               "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons - {"gpu_idle"}),
               "samples": len(self.samples)}
        if self.err:
            out["error"] = self.err
        return out


# ----------------------------------------------------------------------------- jobs

def _bsa():
    import block_sparse_attention_37_b200 as bsa
    bsa.library()
    return bsa


def source_sha():
    h = hashlib.sha256()
    d = os.path.join(ROOT, "block_sparse_attention_37_b200", "csrc")
    for f in ("forward.cu", "tiles.cuh", "attention.cuh", "common.cuh"):
        with open(os.path.join(d, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def traffic_for(key):
    """DRAM bytes per launch from the committed ncu summary, if it matches today's kernel."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(key)
    if not e or e.get("source_sha") != source_sha():
        return None
    return e.get("bytes_per_launch")


class Job:
    """One hot-path instance on one GPU. Subclasses fill in the step.

    End to end (e2e_step): every step first copies that step's inputs from pinned host memory
    into the device buffers the step reads (e2e_inputs), runs the step, and copies its result
    (e2e_output) back to pinned host memory."""
    name = ""
    launches_per_step = 0

    def step(self, ev_fwd=None):  # ev_fwd: (start, end) events around the forward launch
        raise NotImplementedError

    def e2e_inputs(self):
        raise NotImplementedError

    def e2e_output(self):
        raise NotImplementedError

    def e2e_setup(self):
        self.pin = [t.detach().to("cpu").pin_memory() for t in self.e2e_inputs()]
        out = self.e2e_output()
        self.o_host = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        self.h2d = sum(t.numel() * t.element_size() for t in self.pin)
        self.d2h = self.o_host.numel() * self.o_host.element_size()

    def e2e_step(self):
        for dst, src in zip(self.e2e_inputs(), self.pin):
            dst.copy_(src, non_blocking=True)
        self.step()
        self.o_host.copy_(self.e2e_output(), non_blocking=True)


class ArrowJob(Job):
    """MMDiT joint attention with per-head full / arrow / skip modes."""

    def __init__(self, w, dense=False):
        bsa = _bsa()
        self.bsa = bsa
        s = w["shape"]
        self.s = s
        self.dm = bsa.dims(s.B, s.H, s.N, s.d, s.block_q, s.block_k, s.n_text)
        self.host = {"q": w["q"], "k": w["k"], "v": w["v"],
                     "modes": torch.from_numpy(np.zeros_like(w["head_mode"]) if dense else w["head_mode"]),
                     "wins": torch.from_numpy(w["window"]),
                     "cache": w.get("cache")}
        dev = {k: (v.cuda() if v is not None else None) for k, v in self.host.items()}
        self.q, self.k, self.v = dev["q"], dev["k"], dev["v"]
        self.modes, self.wins, self.cache = dev["modes"], dev["wins"], dev["cache"]
        self.blocks = bsa.BlockList.empty(s.B, s.H, s.n_qb, s.n_kb, bitmap=False)
        self.o = torch.empty_like(self.q)
        self.launches_per_step = 2
        self.step()
        torch.cuda.synchronize()
        cnt = self.blocks.cnt.to(torch.int64)
        self.blocks_computed = int(cnt.sum())
        self.blocks_total = s.B * s.H * s.n_qb * s.n_kb
        self.flops = 4.0 * s.block_q * s.block_k * s.d * self.blocks_computed

    def step(self, ev_fwd=None):
        bsa = self.bsa
        bsa.build_mask(self.dm, bsa.MASK_ARROW, self.blocks, head_mode=self.modes, window=self.wins)
        if ev_fwd:
            ev_fwd[0].record()
        bsa.forward(self.dm, self.q, self.k, self.v, self.o, self.modes, blocks=self.blocks, cache_in=self.cache)
        if ev_fwd:
            ev_fwd[1].record()

    def phases(self):
        """The HBM-bound steps beside the forward: the plan search's RSE of this step's output
        against the uncompressed output of the same inputs (every head FULL, computed once
        here), each read once."""
        bsa, s = self.bsa, self.s
        if not hasattr(self, "o_full"):
            self.o_full = torch.empty_like(self.q)
            full = torch.zeros_like(self.modes)
            bsa.forward(self.dm, self.q, self.k, self.v, self.o_full, full)
            self.rse_out = torch.empty(4 * s.H, dtype=torch.float64, device="cuda")
            torch.cuda.synchronize()
        return [("rse", lambda: bsa.rse(self.dm, self.o, self.o_full, self.rse_out), rse_bytes(s.B, s.H, s.N, s.d))]

    def e2e_inputs(self):
        # Q, K, V, the mode table, the windows and (skip heads) the cached fp32 output
        return [t for t in (self.q, self.k, self.v, self.modes, self.wins, self.cache) if t is not None]

    def e2e_output(self):
        return self.o


class ContentJob(Job):
    """FLUX-2048-like pooled top-k selection followed by the sparse forward."""

    def __init__(self, w, dense=False):
        bsa = _bsa()
        self.bsa = bsa
        s = w["shape"]
        self.s = s
        self.dm = bsa.dims(s.B, s.H, s.N, s.d, s.block_q, s.block_k, s.n_text)
        self.q, self.k, self.v = (t.cuda() for t in (w["q"], w["k"], w["v"]))
        self.modes = torch.full((s.H,), 0 if dense else 1, dtype=torch.int32, device="cuda")
        self.spec = bsa.select_spec(bsa.SELECT_POOLED_QK, w["groups"], True)
        self.ws = torch.empty(bsa.select_workspace_size(self.dm, self.spec), dtype=torch.uint8, device="cuda")
        self.blocks = bsa.BlockList.empty(s.B, s.H, s.n_qb, s.n_kb, bitmap=False)
        self.o = torch.empty_like(self.q)
        self.dense = dense
        self.launches_per_step = 3
        self.step()
        torch.cuda.synchronize()
        self.blocks_total = s.B * s.H * s.n_qb * s.n_kb
        self.blocks_computed = self.blocks_total if dense else int(self.blocks.cnt.to(torch.int64).sum())
        self.flops = 4.0 * s.block_q * s.block_k * s.d * self.blocks_computed

    def e2e_inputs(self):
        return [self.q, self.k, self.v]

    def e2e_output(self):
        return self.o

    def fwd_args(self):
        """(dims, Q, K, V, head modes, keyword arguments) of this step's forward."""
        return self.dm, self.q, self.k, self.v, self.modes, {"blocks": self.blocks}

    def phases(self):
        """The HBM-bound steps, each with its algorithmic bytes: pooling reads Q and K once."""
        bsa, s = self.bsa, self.s
        return [("select", lambda: bsa.select_topk(self.dm, self.q, self.k, self.spec, self.blocks, self.ws),
                 select_bytes(s.B, s.H, s.N, s.d))]

    def step(self, ev_fwd=None):
        bsa = self.bsa
        bsa.select_topk(self.dm, self.q, self.k, self.spec, self.blocks, self.ws)
        if ev_fwd:
            ev_fwd[0].record()
        bsa.forward(self.dm, self.q, self.k, self.v, self.o, self.modes, blocks=self.blocks)
        if ev_fwd:
            ev_fwd[1].record()


class DlmJob(Job):
    """SparseD-like: one full-score selection at setup, then forwards reusing the mask."""

    def __init__(self, w, dense=False, n_sets=2):
        bsa = _bsa()
        self.bsa = bsa
        s = w["shape"]
        self.s = s
        self.dm = bsa.dims(s.B, s.H, s.N, s.d, s.block_q, s.block_k, s.n_text)
        self.bias = w["bias"].cuda()
        self.sets = [tuple(t.cuda() for t in W.dlm_step_qkv(s, 3, t)) for t in range(n_sets)]
        self.modes = torch.full((s.H,), 0 if dense else 1, dtype=torch.int32, device="cuda")
        spec = bsa.select_spec(bsa.SELECT_FULL_SCORE, w["groups"], False, s.d ** -0.5)
        ws = torch.empty(bsa.select_workspace_size(self.dm, spec), dtype=torch.uint8, device="cuda")
        self.blocks = bsa.BlockList.empty(s.B, s.H, s.n_qb, s.n_kb, bitmap=False)
        q0, k0, _ = self.sets[0]
        bsa.select_topk(self.dm, q0, k0, spec, self.blocks, ws, bias=self.bias)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        bsa.select_topk(self.dm, q0, k0, spec, self.blocks, ws, bias=self.bias)
        e1.record()
        torch.cuda.synchronize()
        self.selection_ms = e0.elapsed_time(e1)
        self.o = torch.empty_like(q0)
        self.i = 0
        self.launches_per_step = 1
        self.blocks_total = s.B * s.H * s.n_qb * s.n_kb
        self.blocks_computed = self.blocks_total if dense else int(self.blocks.cnt.to(torch.int64).sum())
        self.flops = 4.0 * s.block_q * s.block_k * s.d * self.blocks_computed

    def e2e_inputs(self):
        # the fresh Q, K, V of the next step (the reused block list and the bias stay resident)
        return list(self.sets[self.i % len(self.sets)])

    def e2e_setup(self):
        super().e2e_setup()
        self.pin_sets = [[t.detach().to("cpu").pin_memory() for t in st] for st in self.sets]

    def e2e_step(self):
        for dst, src in zip(self.e2e_inputs(), self.pin_sets[self.i % len(self.sets)]):
            dst.copy_(src, non_blocking=True)
        self.step()
        self.o_host.copy_(self.o, non_blocking=True)

    def e2e_output(self):
        return self.o

    def fwd_args(self):
        q, k, v = self.sets[0]
        return self.dm, q, k, v, self.modes, {"blocks": self.blocks, "bias": self.bias}

    def step(self, ev_fwd=None):
        q, k, v = self.sets[self.i % len(self.sets)]
        self.i += 1
        if ev_fwd:
            ev_fwd[0].record()
        self.bsa.forward(self.dm, q, k, v, self.o, self.modes, blocks=self.blocks, bias=self.bias)
        if ev_fwd:
            ev_fwd[1].record()


class VideoJob(Job):
    """GNA-like 3-D neighborhood attention: permute, mask, forward, unpermute."""

    def __init__(self, w, dense=False):
        bsa = _bsa()
        self.bsa = bsa
        s = w["shape"]
        self.s = s
        g = w["geom"]
        self.geom = bsa.GnaGeom.make(g.grid, g.tile, g.window, g.stride)
        nt = bsa.gna_tiled_len(s.n_text, self.geom)
        self.dm_r = bsa.dims(s.B, s.H, s.N, s.d, s.block_q, s.block_k, s.n_text)
        self.dm = bsa.dims(s.B, s.H, nt, s.d, s.block_q, s.block_k, s.n_text)
        self.raster = [t.cuda() for t in (w["q"], w["k"], w["v"])]
        self.tiled = [torch.empty((s.B, s.H, nt, s.d), dtype=torch.bfloat16, device="cuda") for _ in range(3)]
        self.modes = torch.full((s.H,), 0 if dense else 1, dtype=torch.int32, device="cuda")
        nb = nt // s.block_q
        self.blocks = bsa.BlockList.empty(s.B, s.H, nb, nb, bitmap=False)
        self.o_t = torch.empty_like(self.tiled[0])
        self.o = torch.empty_like(self.raster[0])
        self.launches_per_step = 4
        self.step()
        torch.cuda.synchronize()
        self.blocks_total = s.B * s.H * nb * nb
        self.blocks_computed = int(self.blocks.cnt.to(torch.int64).sum())
        self.flops = 4.0 * s.block_q * s.block_k * s.d * self.blocks_computed
        self.useful_flops = 4.0 * s.d * s.B * s.H * gna_useful_pairs(s.n_text, g.grid, g.window)

    def e2e_inputs(self):
        # raster-order Q, K, V; the result is O in raster order
        return list(self.raster)

    def e2e_output(self):
        return self.o

    def fwd_args(self):
        return self.dm, self.tiled[0], self.tiled[1], self.tiled[2], self.modes, {"blocks": self.blocks,
                                                                                    "gna": self.geom}

    def phases(self):
        """The HBM-bound steps, each with its algorithmic bytes (every row read once, written once)."""
        bsa, s, nt = self.bsa, self.dm_r, self.dm.N
        return [("permute", lambda: bsa.permute_tiles(self.dm_r, self.geom, self.raster, self.tiled),
                 permute_bytes(s.B, s.H, s.N, nt, s.d, 3)),
                ("unpermute", lambda: bsa.unpermute_tiles(self.dm_r, self.geom, [self.o_t], [self.o]),
                 unpermute_bytes(s.B, s.H, s.N, s.d, 1))]

    def step(self, ev_fwd=None):
        bsa = self.bsa
        bsa.permute_tiles(self.dm_r, self.geom, self.raster, self.tiled)
        bsa.build_mask(self.dm, bsa.MASK_GNA, self.blocks, head_mode=self.modes, gna=self.geom)
        if ev_fwd:
            ev_fwd[0].record()
        bsa.forward(self.dm, *self.tiled, self.o_t, self.modes, blocks=self.blocks, gna=self.geom)
        if ev_fwd:
            ev_fwd[1].record()
        bsa.unpermute_tiles(self.dm_r, self.geom, [self.o_t], [self.o])


CONFIGS = {
    "c1": ("tiny arrow: B=1 H=2 d=64 N=512 (64 text + 16x28), block 64, head0 full, head1 arrow w=1",
           lambda seed: W.c1(seed), ArrowJob),
    "c2": ("SD3-1024-like MMDiT joint attention: B=2 H=24 d=64 N=4352 (256 text + 64x64), block 64, "
           "modes 10 full / 11 arrow (w in {1,2,4}) / 3 skip (cached fp32 output)",
           lambda seed: W.c2(seed), ArrowJob),
    "c3": ("FLUX-2048-like pooled selection: B=1 H=24 d=128 N=16896 (512 text + 128x128), block 128, "
           "top-30% image KV blocks + text", lambda seed: W.c3(seed), ContentJob),
    "c4": ("SparseD-like DLM: B=1 H=32 d=128 N=32768 (30720 prefill + 2048 gen), block 128, "
           "isolated top-30% full-score selection reused across steps", lambda seed: W.c4(seed), DlmJob),
    "c5s": ("GNA-like video: B=1 H=24 d=128 256 text + 16x48x80, tile 4x8x8, window 8x16x24, stride 4x8x8",
            lambda seed: W.c5((4, 8, 8), seed), VideoJob),
    "c5f": ("GNA-like video: B=1 H=24 d=128 256 text + 16x48x80, tile 4x8x8, window 8x16x24, stride 1x1x1",
            lambda seed: W.c5((1, 1, 1), seed), VideoJob),
}
DEFAULT_SEEDS = {"c1": 0, "c2": 1, "c3": 2, "c4": 3, "c5s": 4, "c5f": 4}
# (steps, warmup) when not given: about two seconds of timed work per workload
DEFAULT_STEPS = {"c1": (2000, 20), "c2": (2000, 20), "c3": (1000, 20), "c4": (200, 10), "c5s": (500, 10),
                 "c5f": (200, 10)}


# ----------------------------------------------------------------------------- ranks

def rank_seed(cfg: str, rank: int) -> int:
    """Seed of rank `rank`'s independent instance (weak scaling: every rank owns its own batch)."""
    return DEFAULT_SEEDS[cfg] + 1000 * rank


def reduce_sum(vals, world: int, device) -> list:
    """Element-wise sum over ranks (the units of a head-sharded problem)."""
    t = torch.tensor([float(v) for v in vals], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return [float(x) for x in t.tolist()]


def reduce_max(vals, world: int, device) -> list:
    """Element-wise max over ranks (timing only; the data path has no collective)."""
    t = torch.tensor([float(v) for v in vals], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def shard_workload(w, rank: int, world: int):
    """The rank's share of one problem split by heads: every per-head input sliced to the rank's
    contiguous head range (block_sparse_attention_37_b200.sharding)."""
    from block_sparse_attention_37_b200 import sharding
    h0, h1 = sharding.head_range(w["shape"].H, rank, world)
    out = dict(w)
    for key in ("q", "k", "v", "cache"):
        if out.get(key) is not None:
            out[key] = sharding.local_heads(out[key], rank, world)
    for key in ("head_mode", "window"):
        if key in out:
            out[key] = np.ascontiguousarray(out[key][h0:h1])
    if "bias" in out:
        out["bias"] = sharding.local_heads(out["bias"], rank, world, head_dim=0)
    if "bias_kinds" in out:
        out["bias_kinds"] = out["bias_kinds"][h0:h1]
    out["shape"] = W.Shape(**{**out["shape"].__dict__, "H": h1 - h0})
    return out


class HeadShardedJob(Job):
    """One rank's share of a problem split by heads: its heads' whole hot path, then the
    all-gather of O (one NCCL all-gather per batch item) so every rank ends with every head."""

    def __init__(self, job, world):
        self.job, self.world = job, world
        self.s = job.s
        self.launches_per_step = job.launches_per_step
        o = job.e2e_output()
        self.full = torch.empty((o.shape[0], o.shape[1] * world) + tuple(o.shape[2:]), dtype=o.dtype,
                                device=o.device)

    def step(self, ev_fwd=None):
        from block_sparse_attention_37_b200 import sharding
        self.job.step(ev_fwd)
        sharding.gather_heads(self.job.e2e_output(), self.world, out=self.full)

    def e2e_inputs(self):
        return self.job.e2e_inputs()

    def e2e_output(self):
        return self.full

    def e2e_step(self):
        for dst, src in zip(self.e2e_inputs(), self.pin):
            dst.copy_(src, non_blocking=True)
        self.step()
        self.o_host.copy_(self.full, non_blocking=True)


def job_throughput(flops_per_step: float, world: int, ms_per_step: float) -> float:
    """Whole-job TFLOP/s: the units all ranks processed over the slowest rank's time."""
    return flops_per_step * world / (ms_per_step * 1e-3) / 1e12


# ----------------------------------------------------------------------------- HBM-bound phases

def select_bytes(B, H, N, d):
    """Pooled selection: Q and K (bf16) read once; the pooled means and scores stay in L2."""
    return 2 * B * H * N * d * 2


def rse_bytes(B, H, N, d):
    """The plan search's relative squared error: y_m and y_o (bf16) read once."""
    return 2 * B * H * N * d * 2


def permute_bytes(B, H, n_raster, n_tiled, d, n_tensors):
    """Raster -> tile order: every raster row read, every tile-order row (padding too) written."""
    return n_tensors * B * H * (n_raster + n_tiled) * d * 2


def unpermute_bytes(B, H, n_raster, d, n_tensors):
    """Tile order -> raster: the real rows read and written; padding rows are dropped."""
    return n_tensors * B * H * 2 * n_raster * d * 2


def gna_useful_pairs(n_text, grid, window):
    """Allowed (query, key) pairs of one head under the GNA mask: a video query sees exactly the
    product of its per-dimension window lengths (the window is clamped inside the grid) plus the
    text; a text query sees every real token. Padding is neither query nor key."""
    n_img, win = 1, 1
    for L, k in zip(grid, window):
        n_img *= L
        win *= min(k, L)
    return n_img * (win + n_text) + n_text * (n_text + n_img)


def fp8_leg(job, flush, bf16_peak, reps=20, warmup=3):
    """The e4m3 forward (bsa_quantize_fp8 + bsa_forward_fp8) on the operands and block list of the
    job's bf16 forward: the quantisation and the forward each timed alone (CUDA events, L2
    flushed before every call, median of `reps`). Its roofline peak is the measured bf16 peak
    times the nominal 2x of e4m3 over bf16 dense tensor throughput."""
    bsa = job.bsa
    dm, q, k, v, modes, kw = job.fwd_args()
    ops = bsa.Fp8Operands.empty(dm.B, dm.H, dm.N)
    o = torch.empty_like(q)

    def timed(fn):
        for _ in range(warmup):
            flush.zero_()
            fn()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        for e0, e1 in evs:
            flush.zero_()
            e0.record()
            fn()
            e1.record()
        torch.cuda.synchronize()
        return float(np.median([e0.elapsed_time(e1) for e0, e1 in evs]))
    q_ms = timed(lambda: bsa.quantize_fp8(dm, q, k, v, ops))
    f_ms = timed(lambda: bsa.forward_fp8(dm, ops, o, modes, **kw))
    if bsa.get_device_error() != 0:
        raise RuntimeError("device error in the e4m3 forward")
    achieved = job.flops / (f_ms * 1e-3) / 1e12
    peak = 2.0 * bf16_peak
    return {"fwd_ms": f_ms, "fwd_tflops": achieved, "quantize_ms": q_ms,
            "step_tflops_with_quantize": job.flops / ((f_ms + q_ms) * 1e-3) / 1e12,
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "kernel": "bsa::fwd_kernel<128, true> (bsa_forward_fp8)",
                         "peak_source": "measured bf16 burst x 2 (nominal e4m3 / bf16 dense ratio)"}}


def phase_bandwidth(phases, flush, hbm_gbs, reps=20, warmup=3):
    """Each phase timed alone (CUDA events, L2 flushed before every call, median of `reps`),
    as GB/s of its algorithmic bytes against the measured HBM copy bandwidth."""
    out = {}
    for name, fn, nbytes in phases:
        for _ in range(warmup):
            flush.zero_()
            fn()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        for e0, e1 in evs:
            flush.zero_()
            e0.record()
            fn()
            e1.record()
        torch.cuda.synchronize()
        ms = float(np.median([e0.elapsed_time(e1) for e0, e1 in evs]))
        gbs = nbytes / (ms * 1e-3) / 1e9
        out[name] = {"ms": ms, "algorithmic_bytes": int(nbytes), "gbs": gbs, "frac_of_hbm": gbs / hbm_gbs}
    return out


# ----------------------------------------------------------------------------- timing

def time_steps(job, steps, warmup, flush, with_fwd_events=True):
    """Per-step device time (CUDA events on the launching stream), L2 flushed before each step."""
    for _ in range(warmup):
        flush.zero_()
        job.step()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
            torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for e in evs:
        flush.zero_()
        e[0].record()
        job.step((e[2], e[3]) if with_fwd_events else None)
        e[1].record()
    torch.cuda.synchronize()
    step_ms = [e[0].elapsed_time(e[1]) for e in evs]
    fwd_ms = [e[2].elapsed_time(e[3]) for e in evs] if with_fwd_events else None
    return step_ms, fwd_ms


def _blas_threads():
    from threadpoolctl import threadpool_info
    return sum(i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas") or 1


class _Shared:
    """Oracle work that several sampled units use (a head's selection or permutation): done once,
    on first use, with its wall time kept so that each unit can be charged its share."""

    def __init__(self, fn):
        self.fn, self.value, self.seconds = fn, None, None

    def get(self):
        if self.seconds is None:
            t = time.perf_counter()
            self.value = self.fn()
            self.seconds = time.perf_counter() - t
        return self.value


_ORACLE_INPUTS = {}


def _oracle_workload(cfg):
    """The workload's host inputs, drawn once per process (the reference arm samples it per step)."""
    if cfg not in _ORACLE_INPUTS:
        w = CONFIGS[cfg][1](DEFAULT_SEEDS[cfg])
        if cfg == "c4":
            w["steps_qkv"] = (W.dlm_step_qkv(w["shape"], 3, 0), W.dlm_step_qkv(w["shape"], 3, 1))
        _ORACLE_INPUTS[cfg] = w
    return _ORACLE_INPUTS[cfg]


def _oracle_plan(cfg, w, rng):
    """The oracle's work on workload `w`: a seeded random order of units (run, shared, share).

    run() does the unit's oracle work and returns the effective (computed-block) FLOPs of the rows
    it covers, counted like the GPU metric; `shared` (or None) is work the unit needs that it shares
    with other units, and `share` the fraction of that work's time charged to the unit."""
    from oracle import attention as OA
    from oracle import masks as OM
    from oracle import permute as OP
    from oracle import select as OS
    s = w["shape"]
    scale = s.d ** -0.5
    f64 = lambda t: t.double().numpy()
    units = []
    if cfg in ("c1", "c2"):
        # whole heads; the arrow mask is evaluated inside the oracle's forward
        blk = 4.0 * s.block_q * s.block_k * s.d
        for b in range(s.B):
            for h in range(s.H):
                mode, win = int(w["head_mode"][h]), int(w["window"][h])
                if mode == W.HEAD_SKIP:
                    continue

                def run(b=b, h=h, mode=mode, win=win):
                    fn = lambda r: OM.arrow_token_mask(s.N, s.n_text, s.block_q, mode, win, r)
                    OA.head_forward(f64(w["q"][b, h]), f64(w["k"][b, h]), f64(w["v"][b, h]), mode, fn, scale)
                    kept = s.n_qb * s.n_kb if mode == W.HEAD_FULL else \
                        int((OM.arrow_block_classes(s.N, s.n_text, s.block_q, mode, win) > 0).sum())
                    return blk * kept
                units.append((run, None, 0.0))
    elif cfg == "c3":
        # the head's pooled selection (shared by its query blocks), then 4 query blocks per head
        blk = 4.0 * s.block_q * s.block_k * s.d
        for b in range(s.B):
            for h in range(s.H):
                sel = _Shared(lambda b=b, h=h: OS.pooled_select(f64(w["q"][b, h]), f64(w["k"][b, h]), s.block_q,
                                                                s.block_k, s.n_text, w["groups"], True)[0])
                for I in rng.permutation(s.n_qb)[:4]:
                    def run(b=b, h=h, I=int(I), sel=sel):
                        cls = sel.get()
                        rows = np.arange(I * s.block_q, min((I + 1) * s.block_q, s.N))
                        fn = OA.block_mask_to_token_fn(cls, s.block_q, s.block_k, s.N)
                        OA.head_forward(f64(w["q"][b, h]), f64(w["k"][b, h]), f64(w["v"][b, h]), W.HEAD_SPARSE,
                                        fn, scale, rows=rows)
                        return blk * int((cls[I] > 0).sum())
                    units.append((run, sel, 1.0 / s.n_qb))
    elif cfg == "c4":
        # a query block's selection row (A' on step 0, computed once and reused by 8 steps: 1/8 of
        # its time is charged), then one step's forward of the block's rows with the block bias
        blk = 4.0 * s.block_q * s.block_k * s.d
        (q0, k0, _), (q1, k1, v1) = w["steps_qkv"]
        bias = w["bias"].numpy()
        for h in range(s.H):
            for I in rng.permutation(s.n_qb)[:2]:
                def select_row(h=h, I=int(I)):
                    ap = OS.avgpool_attention_rows(f64(q0[0, h]), f64(k0[0, h]), scale, s.block_q, s.block_k, I,
                                                   bias[h])
                    return OS.select_rows(ap[None, :], s.n_kb, w["groups"])[0]
                sel = _Shared(select_row)

                def run(h=h, I=int(I), sel=sel):
                    cls = np.zeros((s.n_qb, s.n_kb), np.uint8)
                    cls[I] = sel.get()
                    rows = np.arange(I * s.block_q, min((I + 1) * s.block_q, s.N))
                    fn = OA.block_mask_to_token_fn(cls, s.block_q, s.block_k, s.N)
                    bfn = OA.block_bias_fn(bias[h], s.block_q, s.block_k, s.N)
                    OA.head_forward(f64(q1[0, h]), f64(k1[0, h]), f64(v1[0, h]), W.HEAD_SPARSE, fn, scale,
                                    rows=rows, bias_fn=bfn)
                    return blk * int((cls[I] > 0).sum())
                units.append((run, sel, 1.0 / 8))
    else:
        # the head's Q, K, V permuted into tile order (shared by its query tiles), then 2 query
        # tiles per head; the GNA mask is evaluated inside the oracle's forward
        g = w["geom"]
        lay = OM.GnaLayout(s.n_text, g.grid, g.tile, g.window, g.stride)
        cls_all = OM.gna_block_classes_separable(lay)
        nb = cls_all.shape[0]
        blk = 4.0 * lay.bs * lay.bs * s.d
        for b in range(s.B):
            for h in range(s.H):
                perm = _Shared(lambda b=b, h=h: [OP.permute_to_tiles(f64(t[b, h]), lay)
                                                 for t in (w["q"], w["k"], w["v"])])
                for I in rng.permutation(nb)[:2]:
                    def run(I=int(I), perm=perm):
                        qt, kt, vt = perm.get()
                        rows = np.arange(I * lay.bs, (I + 1) * lay.bs)
                        rows = rows[lay.valid(rows)]
                        OA.head_forward(qt, kt, vt, W.HEAD_SPARSE, lambda r: OM.gna_token_mask(lay, r), scale,
                                        rows=rows)
                        return blk * int((cls_all[I] > 0).sum())
                    units.append((run, perm, 1.0 / nb))
    order = rng.permutation(len(units))
    return [units[i] for i in order]


ORACLE_SAMPLE = {
    "c1": "(b,h) heads, all rows",
    "c2": "(b,h) heads, all rows",
    "c3": "query blocks, each charged 1/132 of its head's oracle pooled selection",
    "c4": "query blocks of one step's forward, each charged 1/8 of its oracle full-score selection row "
          "(the selection is reused by 8 steps)",
    "c5s": "query tiles, each charged 1/241 of its head's oracle permutation into tile order",
    "c5f": "query tiles, each charged 1/241 of its head's oracle permutation into tile order",
}


def oracle_sample_tflops(cfg, budget_s, seed=0):
    """Time the fp64 oracle on a bounded, seeded sample of the workload (host cores).

    Effective TFLOP/s of the sample: the computed-block FLOPs of the sampled rows over the oracle's
    time for them, shared per-head work charged by the share of the head's rows each unit covers."""
    w = _oracle_workload(cfg)
    units = _oracle_plan(cfg, w, np.random.default_rng(seed))
    flops = charged = 0.0
    done = 0
    t0 = time.perf_counter()
    for run, shared, share in units:
        if shared is not None:
            shared.get()  # timed on its own, charged below by share
        t = time.perf_counter()
        flops += run()
        charged += time.perf_counter() - t + (share * shared.seconds if shared is not None else 0.0)
        done += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    el = time.perf_counter() - t0
    return {"value": flops / charged / 1e12, "unit": UNIT, "cores": int(_blas_threads()), "kind": "oracle",
            "sample": f"{done} of {len(units)} sampled {ORACLE_SAMPLE[cfg]} of the {cfg} workload, "
                      f"{el:.1f} s wall", "seconds": el}


# ----------------------------------------------------------------------------- arms

def run_reference(args, rank, world):
    """--impl reference: the oracle on host cores (rank 0 only)."""
    if rank != 0:
        return 0
    cfg = args.config
    desc = CONFIGS[cfg][0]
    per_step = max(0.2, min(3.0, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample_tflops(cfg, per_step * 0.2)
    vals, secs = [], []
    res = None
    for i in range(args.steps):
        res = oracle_sample_tflops(cfg, per_step, seed=i)
        vals.append(res["value"])
        secs.append(res["seconds"])
    value = float(np.median(vals))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * float(np.mean(secs)),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)",
        "config": {"workload": desc, "impl": "fp64 numpy oracle on host cores"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": res["cores"], "kind": "oracle",
                         "sample": res["sample"]},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_bsa(args, rank, world, local_rank):
    import torch.distributed as dist
    peaks, peak_src = load_peaks()
    cfg = args.config
    desc, make, JobT = CONFIGS[cfg]
    sharded = args.shard == "heads" and world > 1
    seed = DEFAULT_SEEDS[cfg] if sharded else rank_seed(cfg, rank)
    w = make(seed)
    if sharded:
        w = shard_workload(w, rank, world)
        job = HeadShardedJob(JobT(w), world)
    else:
        job = JobT(w)
    inner = job.job if sharded else job
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")

    sampler = ClockSampler(local_rank)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    wall0 = time.perf_counter()
    step_ms, fwd_ms = time_steps(job, args.steps, args.warmup, flush)
    torch.cuda.synchronize()
    wall1 = time.perf_counter()
    sampler.stop()
    if world > 1:
        dist.barrier()
    total_ms, fwd_total = reduce_max([np.sum(step_ms), np.sum(fwd_ms)], world, "cuda")
    ms_per_step = total_ms / args.steps
    fwd_ms_mean = fwd_total / args.steps
    if sharded:  # one problem: the units are the sum of the ranks' shares, over the slowest rank
        flops_all, computed_all, total_all = reduce_sum([inner.flops, inner.blocks_computed,
                                                         inner.blocks_total], world, "cuda")
        value = flops_all / (ms_per_step * 1e-3) / 1e12
    else:
        value = job_throughput(inner.flops, world, ms_per_step)

    extra = {}
    if not args.no_dense:
        dense = JobT(w, dense=True)
        d_step, d_fwd = time_steps(dense, max(10, args.steps // 4), args.warmup, flush)
        sparsity = 1.0 - inner.blocks_computed / inner.blocks_total
        extra = {"dense_fwd_ms": float(np.mean(d_fwd)), "fwd_ms": fwd_ms_mean,
                 "speedup_vs_dense": float(np.mean(d_fwd)) / fwd_ms_mean,
                 "ideal_speedup": 1.0 / (1.0 - sparsity) if sparsity < 1 else None,
                 "block_sparsity": sparsity,
                 "dense_tflops": dense.flops / (float(np.mean(d_fwd)) * 1e-3) / 1e12}
        del dense
    if isinstance(inner, DlmJob):
        extra["selection_ms"] = inner.selection_ms
    if hasattr(inner, "useful_flops"):  # pairs the mask allows, partial tiles counted by their real pairs
        extra["useful_tflops"] = inner.useful_flops / (fwd_ms_mean * 1e-3) / 1e12
        extra["useful_flops_per_step"] = inner.useful_flops
    if not args.no_fp8 and hasattr(inner, "fwd_args") and inner.s.d == 128:
        extra["fp8"] = fp8_leg(inner, flush, peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    if hasattr(inner, "phases"):
        hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
        extra["hbm_phases"] = phase_bandwidth(inner.phases(), flush, hbm)
        extra["hbm_peak_gbs"] = f"{hbm} ({peak_src} copy bandwidth)"

    e2e = None
    if not args.no_e2e:
        job.e2e_setup()
        for _ in range(max(3, args.warmup // 4)):
            job.e2e_step()
        torch.cuda.synchronize()
        n = max(10, min(200, args.steps // 10))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(n):
            job.e2e_step()
        e1.record()
        torch.cuda.synchronize()
        (e2e_ms,) = reduce_max([e0.elapsed_time(e1) / n], world, "cuda")
        e2e_value = flops_all / (e2e_ms * 1e-3) / 1e12 if sharded else job_throughput(inner.flops, world, e2e_ms)
        e2e = {"value": e2e_value, "unit": UNIT,
               "h2d_bytes_per_step": int(job.h2d), "d2h_bytes_per_step": int(job.d2h),
               "ms_per_step": e2e_ms}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = oracle_sample_tflops(cfg, args.cpu_seconds)
        cpu.pop("seconds", None)

    peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    achieved = inner.flops / (fwd_ms_mean * 1e-3) / 1e12
    key = f"attn_fwd_{cfg}"
    roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
            "frac": achieved / peak, "traffic": traffic_for(key),
            "kernel": f"bsa::fwd_kernel<{job.s.d}> (bsa_forward)",
            "peak_source": f"{peak_src} bf16 burst (kernel timed alone between L2 flushes)",
            "algorithmic_flops_per_launch": inner.flops}
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "strong" if sharded else "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded; shapes of the pages' workloads)",
        "config": {"workload": desc, "config": cfg,
                   "l2": "flushed before every step (256 MiB write), flush outside the timed events",
                   "parallelism": (f"one problem split by heads over {world} GPUs, O all-gathered (NCCL) "
                                   "inside every step") if sharded else f"independent replica per GPU x{world}",
                   "seed": DEFAULT_SEEDS[cfg]},
        "pct_of_bf16_peak": 100.0 * value / world / peak,
        "pct_of_bf16_sustained": 100.0 * value / world
        / peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]),
        "roofline": roof,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": inner.launches_per_step * args.steps,
        "clocks": sampler.summary(),
        "wall_s_timed_region": wall1 - wall0,
        "blocks_computed": int(computed_all) if sharded else inner.blocks_computed,
        "blocks_total": int(total_all) if sharded else inner.blocks_total,
    }
    line.update(extra)
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the library has no CPU path)")
    torch.cuda.set_device(local_rank)
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        return run_bsa(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
