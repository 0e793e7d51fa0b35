#!/usr/bin/env python3
"""Benchmark of the Whisper-style attention pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload windows8]
    python bench.py --impl reference ...      # the FP64 CPU oracle on host cores

One step = the whole hot path over one batch: the packed QKV projection
(attn_qkv_pack) followed by multi-head flash attention (attn_forward), for the
8-window encoder workload (8 x 1500 frames, d_model 1280, 20 heads of 64, FULL
mask). Inputs are resident in HBM when the timed region starts; L2 is flushed
(a 256 MiB write) between timed steps, outside the per-step CUDA events. Every
launch is timed with CUDA events on the stream it runs on. With N > 1 (one
process per GPU under torchrun) each rank runs its own 8 windows (weak
scaling, no collective on the data path) and the step time is the maximum
over ranks.

Rank 0 prints one JSON line. `value` is the whole-job throughput in TFLOP/s of
algorithmic QKV + attention flops; `e2e` is the same metric through the same C
ABI calls with the step's input copied from pinned host memory and its output
copied back inside the timed region.
"""
from __future__ import annotations

import argparse
import contextlib
import hashlib
import json
import re
import os
import socket
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from speech_encoder_attention_b200 import inputs  # noqa: E402

METRIC = "attention+QKV TFLOP/s at T=1500, 20x64 heads; % of B200 FP16 tensor peak"
FLUSH_BYTES = 256 << 20
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
KERNEL_SOURCES = ["speech_encoder_attention_b200/csrc/flash_attn.cuh",
                  "speech_encoder_attention_b200/csrc/qkv_gemm.cuh",
                  "speech_encoder_attention_b200/csrc/qkv_q8.cuh",
                  "speech_encoder_attention_b200/csrc/sm100_ptx.cuh",
                  "speech_encoder_attention_b200/csrc/attn_api.cu"]
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ---------------------------------------------------------------------------
# algorithmic work
# ---------------------------------------------------------------------------

def qkv_flops(rows: int, d: int) -> float:
    return 2.0 * rows * d * 3 * d


def attn_pair_flops(pairs: int, heads: int, dh: int = 64) -> float:
    """2*dh flops for the score and 2*dh for the value product, per allowed pair and head."""
    return 4.0 * dh * heads * pairs


def band_pairs(t: int, w: int) -> int:
    """Allowed (query, key) pairs of one t-frame sequence under |i - j| < w."""
    i = np.arange(t)
    return int((np.minimum(t, i + w) - np.maximum(0, i - w + 1)).sum())


def encoder_pairs(spec: inputs.EncoderSpec) -> int:
    if spec.mask == "chunk":
        full, rest = divmod(spec.t, spec.chunk_len)
        return spec.batch * (full * spec.chunk_len ** 2 + rest ** 2)
    if spec.mask == "band":
        return spec.batch * band_pairs(spec.t, spec.band)
    lens = inputs.encoder_lengths(spec)
    if lens is not None:
        return int((lens.astype(np.int64) ** 2).sum())
    return spec.batch * spec.t * spec.t


def encoder_valid_rows(spec: inputs.EncoderSpec) -> int:
    lens = inputs.encoder_lengths(spec)
    return int(lens.sum()) if lens is not None else spec.batch * spec.t


def _strip_comments(src: str) -> str:
    """C/C++ source without its comments and blank lines (string literals in
    these files hold no comment markers)."""
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    return "\n".join(line.rstrip() for line in src.splitlines() if line.strip())


def kernel_source_hash() -> str:
    """Hash of the kernel and launch code (comments excluded): stored ncu
    counters are valid while it is unchanged."""
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), encoding="utf-8") as f:
            h.update(_strip_comments(f.read()).encode())
    return h.hexdigest()[:16]


def load_peaks():
    if os.path.exists(PEAKS_FILE):
        with open(PEAKS_FILE) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def stored_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel sources."""
    try:
        with open(TRAFFIC_FILE) as f:
            doc = json.load(f)
    except (OSError, ValueError):
        return None
    ent = doc.get(workload, {}).get(kernel)
    if not ent or ent.get("source_hash") != kernel_source_hash():
        return None
    return ent.get("dram_bytes_per_launch")


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML reads only)
# ---------------------------------------------------------------------------

REASON_BITS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}


class ClockSampler:
    def __init__(self, device_index: int, period_s: float = 0.001):
        self.period = period_s
        self.samples = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self._nvml = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nvml = None

    def _run(self):
        nv = self._nvml
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                util = nv.nvmlDeviceGetUtilizationRates(self._h).gpu
                try:
                    reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                except AttributeError:
                    reasons = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self._h)
                self.samples.append((sm, util, reasons))
            except Exception:
                pass
            self._stop.wait(self.period)

    def __enter__(self):
        if self._nvml is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0,
                    "note": "no NVML samples"}
        loaded = [s for s in self.samples if s[1] > 0] or self.samples
        mhz = sorted(s[0] for s in loaded)
        bits = 0
        for s in loaded:
            bits |= int(s[2])
        reasons = [name for bit, name in REASON_BITS.items() if bits & bit and name != "gpu_idle"]
        return {"sm_mhz": mhz[len(mhz) // 2], "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(self.samples), "samples_under_load": len(loaded)}


# ---------------------------------------------------------------------------
# distributed plumbing (host side; covered by CPU gloo tests)
# ---------------------------------------------------------------------------

def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def reduce_step_time(local_ms: float, device=None) -> float:
    """Max of the per-rank device-timed step time over all ranks."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return local_ms
    t = torch.tensor([local_ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank_step: float, world: int, ms_per_step: float) -> float:
    """Units all ranks processed per second, at the slowest rank's step time."""
    return units_per_rank_step * world / (ms_per_step * 1e-3)


def relaunch_under_torchrun(n: int, argv):
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__), *argv]
    return subprocess.call(cmd)


# ---------------------------------------------------------------------------
# workloads on the GPU
# ---------------------------------------------------------------------------

class EncoderStep:
    """Packed projection + attention over a batch of windows (or chunks)."""
    cold = False  # L2 flushed before each step; every launch between events

    def __init__(self, spec: inputs.EncoderSpec, device):
        import torch
        from speech_encoder_attention_b200 import attn
        self.attn = attn
        self.spec = spec
        inp = inputs.make_encoder_inputs(spec)
        dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
        self.x, self.w, self.bq, self.bv = dev(inp.x), dev(inp.w_qkv), dev(inp.b_q), dev(inp.b_v)
        rows, d = inp.x.shape
        self.d = d
        self.qkv = torch.empty(rows, 3 * d, dtype=torch.float16, device=device)
        self.out = torch.empty(rows, d, dtype=torch.float16, device=device)
        self.mask = {"chunk": attn.MASK_CHUNK, "band": attn.MASK_BAND}.get(spec.mask, attn.MASK_FULL)
        lens = inputs.encoder_lengths(spec)
        self.lens = None if lens is None else dev(lens)
        self.host_x = torch.from_numpy(inp.x).pin_memory()
        self.host_out = torch.empty(rows, d, dtype=torch.float16).pin_memory()
        self.x_sets = [self.x, self.x.clone()]
        self.out_sets = [self.out, torch.empty_like(self.out)]
        self.host_out_sets = [self.host_out, torch.empty(rows, d, dtype=torch.float16).pin_memory()]
        self.kernels = ["qkv_gemm", "flash_attn"]
        # algorithmic work: the projection of the valid frames, attention over allowed pairs
        self.flops = {"qkv_gemm": qkv_flops(encoder_valid_rows(spec), d),
                      "flash_attn": attn_pair_flops(encoder_pairs(spec), spec.n_heads)}
        self.launches_per_step = 2

    def run(self, events=None, x=None, out=None):
        # Direct launches: a CUDA graph of the two calls measured ~9 us slower
        # per step than these (programmatic launch of the attention grid
        # during the projection's last wave).
        a, d, s = self.attn, self.d, self.spec
        if events:
            events[0].record()
        a.attn_qkv_pack(self.x if x is None else x, self.w, self.bq, self.bv, out=self.qkv)
        if events:
            events[1].record()
        a.attn_forward(self.qkv[:, :d], self.qkv[:, d:2 * d], self.qkv[:, 2 * d:], s.batch, s.t, s.t, s.n_heads,
                       mask_kind=self.mask, chunk_len=s.chunk_len, window=s.band, q_lens=self.lens,
                       kv_lens=self.lens, out=self.out if out is None else out, split=False)
        if events:
            events[2].record()

    # end to end: two sets of input / output buffers (the projection's output
    # is an intermediate of the compute stream alone)
    e2e_sets = 2

    def e2e_in(self, b):
        self.x_sets[b].copy_(self.host_x, non_blocking=True)

    def e2e_compute(self, b):
        self.run(x=self.x_sets[b], out=self.out_sets[b])

    def e2e_out(self, b):
        self.host_out_sets[b].copy_(self.out_sets[b], non_blocking=True)

    def e2e_read_back_matches(self, b):
        return bool((self.host_out_sets[b] == self.out_sets[b].cpu()).all())

    @property
    def h2d_bytes(self):
        return self.host_x.numel() * 2

    @property
    def d2h_bytes(self):
        return self.host_out.numel() * 2

    def total_flops(self):
        return sum(self.flops.values())

    def units(self):
        return {"frames": self.spec.batch * self.spec.t}


class StepGraphs:
    """A decode-side step's library calls captured in CUDA graphs, over N
    device copies of the step's buffers.

    Each copy's step is one graph: its calls back to back, as a decode loop or
    an encoder pipeline captures them (one launch per call, programmatic
    launches between them). A second set of graphs, one per copy and call,
    times the calls one at a time (an event between consecutive calls).

    A decode-side step reads 6-12 MB, far less than the 126 MB L2, so a flush
    write between its steps would also evict the kernels' code and constants,
    which a decode loop finds in L2. Instead such a step's inputs and outputs
    exist N times with N x (bytes of one copy) >= 2 x L2: step i uses copy
    i mod N, whose data was last touched N - 1 steps (more than twice the L2's
    capacity of other data) earlier, so it comes from HBM again."""

    def __init__(self, make_calls, n_copies):
        import torch
        self.n = n_copies
        self.step_graphs, self.call_graphs = [], []
        for i in range(n_copies):
            calls = make_calls(i)
            for fn in calls:  # warm-up: per-device set-up and lazy module loading
                fn()
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for fn in calls:
                    fn()
            self.step_graphs.append(g)
            per_call = []
            for fn in calls:
                gc = torch.cuda.CUDAGraph()
                with torch.cuda.graph(gc):
                    fn()
                per_call.append(gc)
            self.call_graphs.append(per_call)
        torch.cuda.synchronize()
        self.i = 0

    def next_copy(self) -> int:
        i = self.i % self.n
        self.i += 1
        return i

    def run(self, events=None, copy=None):
        """One step on the next copy (or the given one); events = [start, end]."""
        g = self.step_graphs[self.next_copy() if copy is None else copy]
        if events:
            events[0].record()
        g.replay()
        if events:
            events[-1].record()

    def run_split(self, events):
        """One step on the next copy, an event before each call and after the last."""
        graphs = self.call_graphs[self.next_copy()]
        for k, g in enumerate(graphs):
            events[k].record()
            g.replay()
        events[len(graphs)].record()


def cold_copy_count(device, bytes_per_copy: int) -> int:
    import torch
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    return max(2, -(-2 * l2 // max(1, bytes_per_copy)))


STEP_TIMING_COLD = ("each step one CUDA graph; ms_per_step = K steps back to back between two events / K; "
                    "latency_ms_one_step = a second pass with events around each step; per-kernel times = "
                    "a third pass of per-call graphs with an event between calls")
STEP_TIMING_FLUSHED = ("direct launches with an event before, between and after them; L2 flushed before each "
                       "step outside the events")
COLD_L2_NOTE = ("not flushed: inputs and outputs rotate over device copies totalling more than 2 x L2, "
                "so each step reads its data from HBM; one CUDA graph per step")


def cold_note(n_copies: int, bytes_per_copy: int) -> dict:
    return {"copies": n_copies, "bytes_per_copy": bytes_per_copy, "total_bytes": n_copies * bytes_per_copy}


class VerifyStep:
    """Token-tree self-attention (SLOTMASK) plus cross-attention of the same block."""
    cold = True

    def __init__(self, spec: inputs.VerifySpec, device):
        import torch
        from speech_encoder_attention_b200 import attn
        self.attn = attn
        self.spec = spec
        inp = inputs.make_verify_inputs(spec)
        d = spec.d_model
        ws = max(attn.workspace_size(1, spec.t_q, spec.slots, spec.n_heads, attn.MASK_SLOTMASK),
                 attn.workspace_size(1, spec.t_q, spec.t_enc, spec.n_heads, attn.MASK_FULL))
        host = {"q": inp.q, "kc": inp.k_cache, "vc": inp.v_cache, "ke": inp.k_enc, "ve": inp.v_enc,
                "bits": inp.bits.view(np.int32)}
        per_copy = sum(a.nbytes for a in host.values()) + 2 * (2 * spec.t_q * d) + ws
        n = cold_copy_count(device, per_copy)
        self.copies = []
        for _ in range(n):
            c = {k: torch.from_numpy(np.ascontiguousarray(v)).to(device) for k, v in host.items()}
            c["o_self"] = torch.empty(spec.t_q, d, dtype=torch.float16, device=device)
            c["o_cross"] = torch.empty(spec.t_q, d, dtype=torch.float16, device=device)
            c["ws"] = torch.empty(max(ws, 16), dtype=torch.uint8, device=device)
            self.copies.append(c)
        self.cold_copies = cold_note(n, per_copy)
        self.host_q = torch.from_numpy(inp.q).pin_memory()
        self.host_out = torch.empty(2 * spec.t_q, d, dtype=torch.float16).pin_memory()
        pairs = int(inputs.unpack_bits(inp.bits, spec.slots).sum())
        self.kernels = ["slotmask_attn", "cross_attn"]
        self.flops = {"slotmask_attn": attn_pair_flops(pairs, spec.n_heads),
                      "cross_attn": attn_pair_flops(spec.t_q * spec.t_enc, spec.n_heads)}
        b = 2
        self.bytes = {
            "slotmask_attn": b * d * (spec.t_q + 2 * spec.slots + spec.t_q) + 4 * inp.bits.size,
            "cross_attn": b * d * (spec.t_q + 2 * spec.t_enc + spec.t_q),
        }
        # two attention kernels, each followed by a combine kernel unless its
        # key split merges inside a thread-block cluster
        sms = torch.cuda.get_device_properties(device).multi_processor_count
        plans = (attn.debug_plan(1, spec.t_q, spec.slots, spec.n_heads, attn.MASK_SLOTMASK, num_sms=sms),
                 attn.debug_plan(1, spec.t_q, spec.t_enc, spec.n_heads, attn.MASK_FULL, num_sms=sms))
        self.launches_per_step = sum(1 + (pl["kv_splits"] > 1 and not pl["cluster_merge"]) for pl in plans)
        a, s = self.attn, self.spec

        def calls(i):
            c = self.copies[i]
            return [lambda: a.attn_forward(c["q"], c["kc"], c["vc"], 1, s.t_q, s.slots, s.n_heads,
                                           mask_kind=a.MASK_SLOTMASK, bits=c["bits"], out=c["o_self"],
                                           workspace=c["ws"]),
                    lambda: a.attn_cross(c["q"], c["ke"], c["ve"], 1, s.t_q, s.t_enc, s.n_heads, out=c["o_cross"],
                                         workspace=c["ws"])]
        self.graphs = StepGraphs(calls, n)

    def run(self, events=None):
        self.graphs.run(events)

    def run_split(self, events):
        self.graphs.run_split(events)

    # end to end: every device copy is one buffer set
    @property
    def e2e_sets(self):
        return self.graphs.n

    def e2e_in(self, b):
        self.copies[b]["q"].copy_(self.host_q, non_blocking=True)

    def e2e_compute(self, b):
        self.graphs.run(copy=b)

    def e2e_out(self, b):
        self.host_out[:self.spec.t_q].copy_(self.copies[b]["o_self"], non_blocking=True)
        self.host_out[self.spec.t_q:].copy_(self.copies[b]["o_cross"], non_blocking=True)

    def e2e_read_back_matches(self, b):
        import torch
        dev = torch.cat([self.copies[b]["o_self"], self.copies[b]["o_cross"]]).cpu()
        return bool((self.host_out == dev).all())

    @property
    def h2d_bytes(self):
        return self.host_q.numel() * 2

    @property
    def d2h_bytes(self):
        return self.host_out.numel() * 2

    def total_flops(self):
        return sum(self.flops.values())

    def total_bytes(self):
        return sum(self.bytes.values())

    def units(self):
        return {"query_rows": self.spec.t_q}


class DrafterStep:
    """The drafter's block attention: each beam's 16 queries at the end of its
    448 keys, bidirectional or causal inside the block, with per-head sinks."""
    cold = True

    def __init__(self, spec: inputs.DrafterSpec, device):
        import torch
        from speech_encoder_attention_b200 import attn
        self.attn = attn
        self.spec = spec
        inp = inputs.make_drafter_inputs(spec)
        d = spec.d_model
        ws = attn.workspace_size(spec.beams, spec.t_q, spec.t_kv, spec.n_heads, attn.MASK_FULL)
        host = {"q": inp.q, "k": inp.k, "v": inp.v, "sinks": inp.sinks}
        per_copy = sum(a.nbytes for a in host.values()) + 2 * spec.beams * spec.t_q * d + ws
        n = cold_copy_count(device, per_copy)
        self.copies = []
        for _ in range(n):
            c = {k: torch.from_numpy(np.ascontiguousarray(v)).to(device) for k, v in host.items()}
            c["out"] = torch.empty(spec.beams * spec.t_q, d, dtype=torch.float16, device=device)
            c["ws"] = torch.empty(max(ws, 16), dtype=torch.uint8, device=device)
            self.copies.append(c)
        self.cold_copies = cold_note(n, per_copy)
        self.split_launches = 2 if ws > 0 else 1
        self.host_q = torch.from_numpy(inp.q).pin_memory()
        self.host_out = torch.empty(spec.beams * spec.t_q, d, dtype=torch.float16).pin_memory()
        per_beam = (spec.t_q * spec.context + spec.t_q * (spec.t_q + 1) // 2) if spec.causal \
            else spec.t_q * spec.t_kv
        self.kernels = ["drafter_attn"]
        self.flops = {"drafter_attn": attn_pair_flops(spec.beams * per_beam, spec.n_heads)}
        self.bytes = {"drafter_attn": 2 * d * spec.beams * (2 * spec.t_q + 2 * spec.t_kv) + 4 * spec.n_heads}
        self.launches_per_step = self.split_launches
        a, s = self.attn, self.spec

        def calls(i):
            c = self.copies[i]
            return [lambda: a.attn_forward(c["q"], c["k"], c["v"], s.beams, s.t_q, s.t_kv, s.n_heads,
                                           causal=s.causal, sinks=c["sinks"], out=c["out"], workspace=c["ws"])]
        self.graphs = StepGraphs(calls, n)

    def run(self, events=None):
        self.graphs.run(events)

    def run_split(self, events):
        self.graphs.run_split(events)

    @property
    def e2e_sets(self):
        return self.graphs.n

    def e2e_in(self, b):
        self.copies[b]["q"].copy_(self.host_q, non_blocking=True)

    def e2e_compute(self, b):
        self.graphs.run(copy=b)

    def e2e_out(self, b):
        self.host_out.copy_(self.copies[b]["out"], non_blocking=True)

    def e2e_read_back_matches(self, b):
        return bool((self.host_out == self.copies[b]["out"].cpu()).all())

    @property
    def h2d_bytes(self):
        return self.host_q.numel() * 2

    @property
    def d2h_bytes(self):
        return self.host_out.numel() * 2

    def total_flops(self):
        return sum(self.flops.values())

    def total_bytes(self):
        return sum(self.bytes.values())

    def units(self):
        return {"query_rows": self.spec.beams * self.spec.t_q}


class Q8Step:
    """The decoder's packed projection with Q8_0 weights (one launch)."""
    cold = True

    def __init__(self, spec: inputs.Q8Spec, device):
        import torch
        from speech_encoder_attention_b200 import attn
        self.attn = attn
        self.spec = spec
        inp = inputs.make_q8_inputs(spec)
        d = spec.d_model
        host = {"x": inp.x, "w": inp.w_blocks, "bq": inp.b_q, "bv": inp.b_v}
        per_copy = sum(a.nbytes for a in host.values()) + 2 * spec.rows * 3 * d
        n = cold_copy_count(device, per_copy)
        self.copies = []
        for _ in range(n):
            c = {k: torch.from_numpy(np.ascontiguousarray(v)).to(device) for k, v in host.items()}
            c["out"] = torch.empty(spec.rows, 3 * d, dtype=torch.float16, device=device)
            self.copies.append(c)
        self.cold_copies = cold_note(n, per_copy)
        self.host_x = torch.from_numpy(inp.x).pin_memory()
        self.host_out = torch.empty(spec.rows, 3 * d, dtype=torch.float16).pin_memory()
        self.kernels = ["q8_proj"]
        self.flops = {"q8_proj": qkv_flops(spec.rows, d)}
        self.bytes = {"q8_proj": inp.w_blocks.nbytes + 2 * spec.rows * d + 2 * spec.rows * 3 * d}
        self.launches_per_step = 1

        def calls(i):
            c = self.copies[i]
            return [lambda: self.attn.attn_qkv_pack_q8_0(c["x"], c["w"], c["bq"], c["bv"], out=c["out"])]
        self.graphs = StepGraphs(calls, n)

    def run(self, events=None):
        self.graphs.run(events)

    def run_split(self, events):
        self.graphs.run_split(events)

    @property
    def e2e_sets(self):
        return self.graphs.n

    def e2e_in(self, b):
        self.copies[b]["x"].copy_(self.host_x, non_blocking=True)

    def e2e_compute(self, b):
        self.graphs.run(copy=b)

    def e2e_out(self, b):
        self.host_out.copy_(self.copies[b]["out"], non_blocking=True)

    def e2e_read_back_matches(self, b):
        return bool((self.host_out == self.copies[b]["out"].cpu()).all())

    @property
    def h2d_bytes(self):
        return self.host_x.numel() * 2

    @property
    def d2h_bytes(self):
        return self.host_out.numel() * 2

    def total_flops(self):
        return sum(self.flops.values())

    def total_bytes(self):
        return sum(self.bytes.values())

    def units(self):
        return {"rows": self.spec.rows}


def make_step(name, device):
    if name in inputs.Q8_WORKLOADS:
        return Q8Step(inputs.Q8_WORKLOADS[name], device)
    if name in inputs.ENCODER_WORKLOADS:
        return EncoderStep(inputs.ENCODER_WORKLOADS[name], device)
    if name in inputs.DRAFTER_WORKLOADS:
        return DrafterStep(inputs.DRAFTER_WORKLOADS[name], device)
    return VerifyStep(inputs.VERIFY_WORKLOADS[name], device)


# ---------------------------------------------------------------------------
# oracle timing (host cores): the reference arm and the cpu_baseline leg
# ---------------------------------------------------------------------------

def oracle_sample(spec: inputs.EncoderSpec, inp, i: int):
    """One bounded sample of the encoder workload: window i % batch, head
    i % n_heads -- that head's slice of the packed projection (q, k, v columns)
    and its attention over the window, by the FP64 oracle. Returns flops."""
    import oracle
    d, t = spec.d_model, spec.t
    b, h = i % spec.batch, i % spec.n_heads
    cols = np.r_[h * 64:(h + 1) * 64, d + h * 64:d + (h + 1) * 64, 2 * d + h * 64:2 * d + (h + 1) * 64]
    lens = inputs.encoder_lengths(spec)
    n = t if lens is None else int(lens[b])  # valid frames of the window
    x = inp.x[b * t:b * t + n]
    qkv = oracle.qkv_projection(x, inp.w_qkv[cols], inp.b_q[h * 64:(h + 1) * 64], inp.b_v[h * 64:(h + 1) * 64])
    if spec.mask == "chunk":
        allowed = oracle.allowed_chunk(n, spec.chunk_len)
    else:
        allowed = oracle.allowed_range(n, n, window=spec.band)
    oracle.attention(qkv[:, :64], qkv[:, 64:128], qkv[:, 128:], 1, allowed)
    return 2.0 * n * d * 192 + attn_pair_flops(int(allowed.sum()), 1)


def oracle_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info()]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count() or 1


def time_oracle(spec, seconds: float = 10.0, max_samples: int = 400):
    inp = inputs.make_encoder_inputs(spec)
    oracle_sample(spec, inp, 0)  # warm
    t0 = time.perf_counter()
    flops, n = 0.0, 0
    while n < max_samples and (time.perf_counter() - t0 < seconds or n == 0):
        flops += oracle_sample(spec, inp, n)
        n += 1
    el = time.perf_counter() - t0
    return {"value": flops / el / 1e12, "unit": "TFLOP/s", "cores": oracle_threads(), "kind": "oracle",
            "sample": f"{n} samples of (one window x one head) of {spec.name}: that head's 192 packed-projection "
                      f"columns over {spec.t} frames plus its attention, NumPy float64, {el:.1f} s"}


def workload_spec(name):
    for table in (inputs.ENCODER_WORKLOADS, inputs.VERIFY_WORKLOADS, inputs.DRAFTER_WORKLOADS,
                  inputs.Q8_WORKLOADS):
        if name in table:
            return table[name]
    raise KeyError(name)


def workload_metric(spec) -> str:
    if isinstance(spec, inputs.EncoderSpec):
        return METRIC
    if isinstance(spec, inputs.DrafterSpec):
        return "drafter block attention TFLOP/s (HBM-bound; see roofline)"
    if isinstance(spec, inputs.Q8Spec):
        return "Q8_0 packed projection TFLOP/s (HBM-bound; see roofline)"
    return "verify+cross attention TFLOP/s (HBM-bound; see roofline)"


class SmallOracleStep:
    """The whole verify or drafter step in FP64 (small enough to run entire)."""

    def __init__(self, spec):
        self.spec = spec
        if isinstance(spec, inputs.DrafterSpec):
            self.inp = inputs.make_drafter_inputs(spec)
        elif isinstance(spec, inputs.Q8Spec):
            self.inp = inputs.make_q8_inputs(spec)
        else:
            self.inp = inputs.make_verify_inputs(spec)

    def __call__(self, i=0) -> float:
        import oracle
        s, inp = self.spec, self.inp
        if isinstance(s, inputs.Q8Spec):
            oracle.qkv_projection_q8_0(inp.x, inp.w_blocks, inp.b_q, inp.b_v)
            return qkv_flops(s.rows, s.d_model)
        if isinstance(s, inputs.DrafterSpec):
            oracle.range_attention(inp.q, inp.k, inp.v, s.beams, s.t_q, s.t_kv, s.n_heads, causal=s.causal,
                                   sinks=inp.sinks)
            a = oracle.allowed_range(s.t_q, s.t_kv, causal=s.causal)
            return attn_pair_flops(s.beams * int(a.sum()), s.n_heads)
        oracle.slotmask_attention(inp.q, inp.k_cache, inp.v_cache, inp.bits, s.n_heads)
        oracle.cross_attention(inp.q, inp.k_enc, inp.v_enc, s.n_heads)
        pairs = int(inputs.unpack_bits(inp.bits, s.slots).sum()) + s.t_q * s.t_enc
        return attn_pair_flops(pairs, s.n_heads)

    def describe(self, n, el):
        return (f"{n} runs of the whole {self.spec.name} step (every row and head), NumPy float64, {el:.1f} s")


def time_small_oracle(spec, seconds: float = 10.0, max_runs: int = 200):
    run = SmallOracleStep(spec)
    run()
    t0 = time.perf_counter()
    flops, n = 0.0, 0
    while n < max_runs and (time.perf_counter() - t0 < seconds or n == 0):
        flops += run(n)
        n += 1
    el = time.perf_counter() - t0
    return {"value": flops / el / 1e12, "unit": "TFLOP/s", "cores": oracle_threads(), "kind": "oracle",
            "sample": run.describe(n, el)}


def run_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    spec = workload_spec(args.workload)
    if isinstance(spec, inputs.EncoderSpec):
        inp = inputs.make_encoder_inputs(spec)
        sample = lambda i: oracle_sample(spec, inp, i)
        what = ("each step: one window x one head of the workload (that head's packed-projection columns "
                "and its attention), FP64 oracle on host cores")
    else:
        sample = SmallOracleStep(spec)
        what = "each step: the whole workload (every row and head), FP64 oracle on host cores"
    for i in range(args.warmup):
        sample(i)
    t0 = time.perf_counter()
    flops = 0.0
    for i in range(args.steps):
        flops += sample(i)
    el = time.perf_counter() - t0
    value = flops / el / 1e12
    line = {
        "impl": "reference", "metric": workload_metric(spec), "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)",
        "config": workload_config(spec),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle_threads(), "kind": "oracle",
                         "sample": what},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(spec):
    if isinstance(spec, inputs.EncoderSpec):
        lens = inputs.encoder_lengths(spec)
        wl = (f"{spec.name}: {spec.batch} x {spec.t}-frame sequence(s), d_model {spec.d_model}, "
              f"{spec.n_heads}x64 heads, {spec.mask.upper()} mask"
              + (f" (chunks of {spec.chunk_len})" if spec.mask == "chunk" else "")
              + (f" (window {spec.band})" if spec.mask == "band" else "")
              + (f", valid lengths {lens.tolist()}" if lens is not None else ""))
        cfg = {"workload": wl, "batch": spec.batch, "t": spec.t, "d_model": spec.d_model,
               "n_heads": spec.n_heads, "head_dim": 64, "mask": spec.mask,
               "l2": "flushed between timed steps (256 MiB write)", "parallelism": "replicas (weak)"}
        if lens is not None:
            cfg["valid_lengths"] = lens.tolist()
        if spec.mask == "band":
            cfg["window"] = spec.band
        return cfg
    if isinstance(spec, inputs.Q8Spec):
        return {"workload": f"{spec.name}: packed projection of {spec.rows} decoder rows, d_model {spec.d_model}, "
                            f"Q8_0 weights [{3 * spec.d_model} x {spec.d_model}]",
                "rows": spec.rows, "d_model": spec.d_model, "weights": "Q8_0 (34-byte blocks)",
                "l2": COLD_L2_NOTE, "parallelism": "replicas (weak)"}
    if isinstance(spec, inputs.DrafterSpec):
        return {"workload": f"{spec.name}: {spec.beams} beams x {spec.t_q} queries at the end of {spec.t_kv} keys, "
                            f"{'causal' if spec.causal else 'bidirectional'} block, per-head sinks, "
                            f"{spec.n_heads}x64 heads",
                "beams": spec.beams, "t_q": spec.t_q, "t_kv": spec.t_kv, "causal": spec.causal,
                "n_heads": spec.n_heads, "l2": COLD_L2_NOTE,
                "parallelism": "replicas (weak)"}
    return {"workload": f"{spec.name}: {spec.t_q} query rows ({spec.beams} beams x {spec.block}) over a "
                        f"{spec.slots}-slot token-tree cache + cross-attention to {spec.t_enc} encoder frames",
            "t_q": spec.t_q, "slots": spec.slots, "t_enc": spec.t_enc, "n_heads": spec.n_heads,
            "l2": COLD_L2_NOTE, "parallelism": "replicas (weak)"}


# ---------------------------------------------------------------------------
# the GPU arm
# ---------------------------------------------------------------------------

def check_device_errors(step, where):
    """A kernel whose bounded wait expired gave up (its output is void) and
    recorded it in the library's device error word: such a run measures nothing."""
    st, word = step.attn.debug_error_word()
    if st != step.attn.ATTN_OK or word != 0:
        raise RuntimeError(f"device error word {word:#x} after the {where}: a kernel wait timed out")


def time_steps(step, flush, steps, warmup, clocks=None, barrier=None):
    """Warm-up, then `steps` timed steps.

    step.cold (a decode-side step: one CUDA graph per step, buffers rotating
    over copies larger than L2, no flush): the K steps run back to back
    between two events, as the base contract times them; a second pass
    brackets each step with its own events (the latency of one step, graph
    launch included); a third replays per-call graphs with an event between
    calls (the per-kernel times).
    Otherwise (the encoder): L2 is flushed (a 256 MiB write) before each step,
    outside its events, and an event sits before, between and after the
    step's launches.
    Returns (mean step ms, [mean ms per kernel], mean one-step latency ms or None)."""
    import torch
    cold = getattr(step, "cold", False)
    nk = len(step.kernels)
    new_events = lambda n: [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    for _ in range(warmup):
        if not cold:
            flush.zero_()
        step.run()
        if cold:
            step.run_split(new_events(nk + 1))
    torch.cuda.synchronize()
    block = new_events(2)
    ev = [new_events(2 if cold else nk + 1) for _ in range(steps)]
    if barrier is not None:
        barrier()
    torch.cuda.synchronize()
    with (clocks if clocks is not None else contextlib.nullcontext()):
        if cold:
            block[0].record()
            for _ in range(steps):
                step.run()
            block[1].record()
        else:
            for e in ev:
                flush.zero_()
                step.run(e)
        torch.cuda.synchronize()
    if barrier is not None:
        barrier()
    if not cold:
        step_ms = sum(e[0].elapsed_time(e[-1]) for e in ev) / steps
        per_kernel = [sum(e[k].elapsed_time(e[k + 1]) for e in ev) / steps for k in range(nk)]
        return step_ms, per_kernel, None
    step_ms = block[0].elapsed_time(block[1]) / steps
    for e in ev:
        step.run(e)
    torch.cuda.synchronize()
    latency_ms = sum(e[0].elapsed_time(e[1]) for e in ev) / steps
    ev = [new_events(nk + 1) for _ in range(steps)]
    for e in ev:
        step.run_split(e)
    torch.cuda.synchronize()
    per_kernel = [sum(e[k].elapsed_time(e[k + 1]) for e in ev) / steps for k in range(nk)]
    return step_ms, per_kernel, latency_ms


def time_e2e(step, steps, warmup, barrier=None):
    """End-to-end steps through the same library calls with host buffers.
    Step i copies its input from pinned host memory into buffer set i mod B
    on a copy-in stream, runs its calls on the compute stream once that copy
    has landed, and reads its result back into pinned host memory on a
    copy-out stream once they are done. A set is written again only after
    the step that used it B steps earlier has been computed (input) and read
    back (output), so neighbouring steps' copies overlap the compute, as a
    streaming pipeline runs them. Timed from before the first copy to after
    the last read-back. Returns ms per step."""
    import torch
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    nb = step.e2e_sets
    ev = lambda: torch.cuda.Event()
    in_done, comp_done, out_done = [ev() for _ in range(nb)], [ev() for _ in range(nb)], [ev() for _ in range(nb)]

    def run(n):
        s_in.wait_stream(comp)
        for i in range(n):
            b = i % nb
            with torch.cuda.stream(s_in):
                if i >= nb:
                    s_in.wait_event(comp_done[b])  # the step that read this input set is done
                step.e2e_in(b)
                in_done[b].record(s_in)
            comp.wait_event(in_done[b])
            if i >= nb:
                comp.wait_event(out_done[b])  # this output set has been read back
            step.e2e_compute(b)
            comp_done[b].record(comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(comp_done[b])
                step.e2e_out(b)
                out_done[b].record(s_out)
        comp.wait_stream(s_out)
        comp.wait_stream(s_in)

    run(max(1, warmup))
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if barrier is not None:
        barrier()
    torch.cuda.synchronize()
    start.record(comp)
    run(steps)
    end.record(comp)
    torch.cuda.synchronize()
    if barrier is not None:
        barrier()
    # the last read-back holds the last step's result
    if not step.e2e_read_back_matches((steps - 1) % nb):
        raise RuntimeError("end-to-end read-back differs from the device result: stream ordering is broken")
    return start.elapsed_time(end) / steps


def time_secondary(name, device, steps, warmup, ws):
    """The bandwidth-bound verify step (token-tree SLOTMASK + cross-attention),
    timed like a `--workload verify` run (data cold in HBM, CUDA events on the
    launching stream, max over ranks): its step time, algorithmic bytes and
    fraction of the HBM roofline."""
    import torch
    step = make_step(name, device)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)
    local_ms, per_kernel, latency_ms = time_steps(step, flush, steps, warmup)
    check_device_errors(step, f"{name} steps")
    ms = reduce_step_time(local_ms, device)
    latency_ms = reduce_step_time(latency_ms, device)
    peaks, peak_kind = load_peaks()
    total_bytes = step.total_bytes()
    gbs = total_bytes / (ms * 1e-3) / 1e9
    return {"workload": workload_config(step.spec)["workload"], "ms_per_step": ms,
            "algorithmic_bytes_per_step": total_bytes, "achieved_gbs": gbs, "peak_gbs": peaks["hbm_gbs"],
            "hbm_frac": gbs / peaks["hbm_gbs"], "peak_source": f"{peak_kind} hbm_gbs",
            "tflops": step.total_flops() / (ms * 1e-3) / 1e12,
            "kernels_us": {k: per_kernel[i] * 1e3 for i, k in enumerate(step.kernels)},
            "latency_ms_one_step": latency_ms,
            "launches_per_step": step.launches_per_step, "cold_copies": step.cold_copies,
            "timing": STEP_TIMING_COLD}


def run_gpu(args):
    import torch
    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if ws > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)
    step = make_step(args.workload, device)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)

    def barrier():
        if ws > 1:
            import torch.distributed as dist
            dist.barrier()

    clocks = ClockSampler(local)
    local_ms, per_kernel, latency_ms = time_steps(step, flush, args.steps, args.warmup, clocks, barrier)
    check_device_errors(step, "timed steps")
    per_kernel = np.asarray(per_kernel)
    ms = reduce_step_time(local_ms, device)
    if latency_ms is not None:
        latency_ms = reduce_step_time(latency_ms, device)

    # end to end through the same calls, host buffers, copies inside the timed region
    e2e_ms = None
    if not args.skip_e2e:
        n_e2e = max(1, min(args.steps, args.e2e_steps))
        e2e_local = time_e2e(step, n_e2e, max(2, args.warmup // 2), barrier)
        check_device_errors(step, "end-to-end steps")
        e2e_ms = reduce_step_time(e2e_local, device)

    # the bandwidth-bound decoder step, reported beside the encoder headline
    secondary = None
    if isinstance(step, EncoderStep) and not args.skip_secondary:
        secondary = time_secondary("verify", device, max(args.steps, 50), max(args.warmup, 3), ws)

    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank != 0:
        return 0

    peaks, peak_kind = load_peaks()
    spec = step.spec
    is_encoder = isinstance(step, EncoderStep)
    flops = step.total_flops()
    value = whole_job_rate(flops, ws, ms) / 1e12
    top = int(np.argmax(per_kernel))
    kname = step.kernels[top]
    clock_rec = clocks.summary()
    # The burst peak for a kernel timed in a short run, the sustained one
    # (a seconds-long loop under the power cap) once the power cap acted
    # during the timed steps.
    capped = "sw_power_cap" in (clock_rec or {}).get("reasons", [])
    tensor_key = "bf16_tflops_sustained" if capped and "bf16_tflops_sustained" in peaks else "bf16_tflops"
    if is_encoder:
        peak = peaks[tensor_key]
        achieved = step.flops[kname] / (per_kernel[top] * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "frac_of_burst_peak": achieved / peaks["bf16_tflops"],
                "traffic": stored_traffic(kname, args.workload), "kernel": kname,
                "peak_source": (f"{peak_kind} {tensor_key} "
                                + ("(sustained: sw_power_cap active during the timed steps)" if capped
                                   else "(burst)") + "; fp16 dense rate = bf16 rate"),
                "algorithmic_flops_per_launch": step.flops[kname], "launch_us": per_kernel[top] * 1e3}
        unit = "TFLOP/s"
    else:
        peak = peaks["hbm_gbs"]
        achieved = step.bytes[kname] / (per_kernel[top] * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                "traffic": stored_traffic(kname, args.workload), "kernel": kname,
                "peak_source": f"{peak_kind} hbm_gbs", "algorithmic_bytes_per_launch": step.bytes[kname],
                "launch_us": per_kernel[top] * 1e3}
        unit = "TFLOP/s"
    metric = workload_metric(spec)
    all_kernels = {}
    for k, name in enumerate(step.kernels):
        ent = {"launch_us": per_kernel[k] * 1e3,
               "tflops": step.flops[name] / (per_kernel[k] * 1e-3) / 1e12}
        if not is_encoder:
            ent["gbs"] = step.bytes[name] / (per_kernel[k] * 1e-3) / 1e9
        all_kernels[name] = ent
    cpu = None
    if not args.skip_cpu_baseline and ws == 1:  # the host baseline is an N = 1 figure
        cpu = (time_oracle(spec, seconds=args.cpu_seconds) if is_encoder
               else time_small_oracle(spec, seconds=args.cpu_seconds))
    line = {
        "metric": metric, "value": value, "unit": unit, "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16", "data": "synthetic (seeded; random-init weights)",
        "config": workload_config(spec),
        "pct_of_peak": 100.0 * value / (peaks["bf16_tflops"] * ws),
        **({"pct_of_sustained_peak": 100.0 * value / (peaks["bf16_tflops_sustained"] * ws)}
           if is_encoder and "bf16_tflops_sustained" in peaks else {}),
        "units_per_s": {k: v * ws / (ms * 1e-3) for k, v in step.units().items()},
        "roofline": roof,
        "kernels": all_kernels,
        "cpu_baseline": cpu,
        "e2e": None if e2e_ms is None else {
            "value": whole_job_rate(flops, ws, e2e_ms) / 1e12, "unit": unit,
            "h2d_bytes_per_step": step.h2d_bytes, "d2h_bytes_per_step": step.d2h_bytes,
            "ms_per_step": e2e_ms,
            "timing": ("steps pipelined over a copy-in, a compute and a copy-out stream with "
                       f"{step.e2e_sets} buffer sets; pinned host memory; first copy to last read-back")},
        "secondary": secondary,
        "gpu_launches": step.launches_per_step * args.steps,
        "timing": STEP_TIMING_COLD if getattr(step, "cold", False) else STEP_TIMING_FLUSHED,
        **({"cold_copies": step.cold_copies, "latency_ms_one_step": latency_ms}
           if getattr(step, "cold", False) else {}),
        "clocks": clock_rec,
        "kernel_source_hash": kernel_source_hash(),
    }
    print(json.dumps(line), flush=True)
    return 0


def parse(argv=None):
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=2000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", choices=["native", "reference"], default="native")
    p.add_argument("--workload", default="windows8",
                   choices=sorted(inputs.ENCODER_WORKLOADS) + sorted(inputs.VERIFY_WORKLOADS)
                   + sorted(inputs.DRAFTER_WORKLOADS) + sorted(inputs.Q8_WORKLOADS))
    p.add_argument("--e2e-steps", type=int, default=200)
    p.add_argument("--cpu-seconds", type=float, default=10.0)
    p.add_argument("--skip-cpu-baseline", action="store_true")
    p.add_argument("--skip-e2e", action="store_true")
    p.add_argument("--skip-secondary", action="store_true",
                   help="do not time the verify step beside an encoder workload")
    args = p.parse_args(argv)
    if args.warmup < 3 and args.impl == "native":
        p.error("--warmup must be at least 3")
    return args


def main(argv=None):
    argv = sys.argv[1:] if argv is None else argv
    args = parse(argv)
    ws, _, _ = dist_env()
    if args.impl == "reference":
        return run_reference(args)
    if args.gpus > 1 and ws == 1:
        return relaunch_under_torchrun(args.gpus, argv)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
