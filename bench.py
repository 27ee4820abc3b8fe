#!/usr/bin/env python
"""Throughput of the attention hot path on B200, one JSON line on rank 0.

A step is one pass of the whole hot path over one batch of synthetic inputs:
  * the seqlen sweep at hidden 2048 (H=32,D=64 and H=16,D=128; S = 512..16k,
    B = 16384/S; causal and non-causal; bf16): forward + backward of each point;
  * the GQA + local-attention workload (B=2, S=4096, Hq=32, Hkv=8, D=128,
    window (1024,0), softcap 30): forward + backward, once with atomic and
    once with deterministic (ordered) dQ accumulation;
  * the paged KV-cache decode (B=8, Hq=32, Hkv=8, D=128, lengths U[1,32768],
    page 256): append + split-KV attention + combine, with the automatic
    split count and with 1, 4 and 16 splits.
``value`` is algorithmic attention TFLOP/s of the whole step (4*D flops per
visible (query, key) pair forward, 10*D backward; decode flops counted the
same way) with inputs resident in HBM.  ``per_config`` gives, from CUDA
events around every API call of the timed steps, each point's forward and
forward+backward TFLOP/s as fractions of the measured bf16 tensor rates and
each decode call's GB/s as a fraction of the measured HBM copy rate;
``per_config_summary`` the worst head-dim-128 point at S >= 4096 and the
worst decode call.  Every tensor of a sweep point, the GQA
workload and the KV cache is larger than L2 (126 MB per step working set far
exceeds it), so L2 is not flushed; before the first decode call of the full
step a 256 MB read writes back the dirty lines the backward left (inside the
step time, outside the decode call's span).  Multi-GPU: every rank runs its own replica
of the step (the work units are independent), value sums all ranks' flops
over the max time across ranks.
"""

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

METRIC = "attention TFLOPs/s fwd & fwd+bwd at seqlen 512–16k, d64/128 (% of tensor peak)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# Launch whose per-launch roofline is reported for each kernel class.
ROOFLINE_UNIT = {"fwd": "H16D128S4096n", "bwd": "H16D128S4096n", "fwd8": "fp8-H16D128S4096n", "decode": "decode"}
# dense E4M3 tensor throughput over bf16 (nominal 4.5 / 2.25 PFLOP/s): the FP8
# roofline peak is the measured bf16 figure times this ratio
FP8_OVER_BF16 = 2.0
# DRAM bytes (read + write) per launch from one ncu capture of that launch
# (profiles/fwd_tc_kernel_H16D128S4096n.md, profiles/bwd_tc_kernel_H16D128S4096n.md,
# profiles/decode_tma_kernel_paged_B8.md).  An entry must be removed whenever
# its kernel changes.
TRAFFIC_PER_LAUNCH = {
    ("fwd", "H16D128S4096n"): 201.659904e6 + 51.587840e6,
    ("bwd", "H16D128S4096n"): 422.807296e6 + 244.183296e6,
    ("decode", "decode"): 521.979136e6 + 5.864960e6,
}


# ---------------------------------------------------------------------------
# algorithmic work
# ---------------------------------------------------------------------------

def visible_pairs(Sq, Sk, causal, wl, wr):
    """Number of visible (query, key) pairs of one head (bottom-right aligned)."""
    if causal:
        wr = 0
    i = np.arange(Sq, dtype=np.int64) + (Sk - Sq)
    lo = np.maximum(0, i - wl) if wl >= 0 else np.zeros_like(i)
    hi = np.minimum(Sk - 1, i + wr) if wr >= 0 else np.full_like(i, Sk - 1)
    return int(np.maximum(0, hi - lo + 1).sum())


def attn_flops(cfg):
    pairs = visible_pairs(cfg["Sq"], cfg["Sk"], cfg["causal"], cfg["window"][0], cfg["window"][1])
    n = pairs * cfg["B"] * cfg["Hq"]
    return 4 * cfg["D"] * n, 10 * cfg["D"] * n


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu_index = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"fa_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader",
                                          "-lms", "200", "-i", str(self.gpu_index)],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append(dict(sm=float(parts[1].split()[0]), smax=float(parts[2].split()[0]),
                                     power=float(parts[3].split()[0]) if parts[3][0].isdigit() else 0.0,
                                     hw=parts[5], hwt=parts[6], swt=parts[7], swp=parts[8]))
                except (ValueError, IndexError):
                    continue
        os.unlink(self.path)
        if not rows:
            return None
        reasons = set()
        for r in rows:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("swp", "sw_power_cap")):
                if r[key].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in rows), "sm_max_mhz": max(r["smax"] for r in rows),
                "samples": len(rows), "reasons": sorted(reasons)}


# ---------------------------------------------------------------------------
# workload units
# ---------------------------------------------------------------------------

class AttnUnit:
    kind = "attn"

    def __init__(self, cfg, dev, deterministic=False):
        from exact_attention_121_b200 import api, inputs
        self.api = api
        self.cfg = cfg
        self.det = deterministic
        q, k, v, do = inputs.attention_inputs(cfg["B"], cfg["Sq"], cfg["Sk"], cfg["Hq"], cfg["Hkv"], cfg["D"],
                                              cfg["dtype"], seed=cfg["seed"], amp=cfg.get("amp", 1.0))
        self.host_in = (q, k, v, do)
        self.q, self.k, self.v, self.do = (t.to(dev) for t in (q, k, v, do))
        self.out = torch.empty_like(self.q)
        self.lse = torch.empty(cfg["B"], cfg["Hq"], cfg["Sq"], device=dev)
        self.dq, self.dk, self.dv = torch.empty_like(self.q), torch.empty_like(self.k), torch.empty_like(self.v)
        n = api.fa_bwd_workspace_size(cfg["B"], cfg["Sq"], cfg["Sk"], cfg["Hq"], cfg["Hkv"], cfg["D"], self.det)
        self.ws = torch.empty(n, dtype=torch.uint8, device=dev)
        self.flops_fwd, self.flops_bwd = attn_flops(cfg)
        self.kw = dict(scale=cfg["scale"], causal=cfg["causal"], window=cfg["window"], softcap=cfg["softcap"])
        if cfg.get("alibi"):
            self.kw["alibi_slopes"] = inputs.alibi_slopes(cfg["Hq"]).to(dev)

    def name(self):
        c = self.cfg
        return "H%dD%dS%d%s%s%s" % (c["Hq"], c["D"], c["Sq"], "c" if c["causal"] else "n", "-det" if self.det else "",
                                    "-alibi" if c.get("alibi") else "")

    def run(self, tracer):
        api = self.api
        tracer.arm("fwd", self)
        api.fa_fwd(self.q, self.k, self.v, out=self.out, lse=self.lse, **self.kw)
        n = api.fa_last_launch_count()
        tracer.arm("bwd", self)
        api.fa_bwd(self.do, self.q, self.k, self.v, self.out, self.lse, self.dq, self.dk, self.dv,
                   deterministic=self.det, workspace=self.ws, **self.kw)
        tracer.disarm()
        return n + api.fa_last_launch_count()

    def flops(self):
        return self.flops_fwd + self.flops_bwd

    # end-to-end: inputs from pinned host memory, outputs back to pinned host memory
    def setup_e2e(self, pinned):
        self.pin_in = [pinned.get(t, i) for i, t in enumerate(self.host_in)]
        self.pin_out = [pinned.get_like(t) for t in (self.out, self.dq, self.dk, self.dv)]

    def copy_in(self):
        for dst, src in zip((self.q, self.k, self.v, self.do), self.pin_in):
            dst.copy_(src, non_blocking=True)

    def copy_out(self):
        for dst, src in zip(self.pin_out, (self.out, self.dq, self.dk, self.dv)):
            dst.copy_(src, non_blocking=True)

    def e2e_bytes(self):
        return (sum(t.numel() * t.element_size() for t in (self.q, self.k, self.v, self.do)),
                sum(t.numel() * t.element_size() for t in (self.out, self.dq, self.dk, self.dv)))


class VarlenUnit(AttnUnit):
    """Packed variable-length batch: forward + backward through the varlen calls."""

    def __init__(self, cfg, dev):
        from exact_attention_121_b200 import api, inputs
        self.api = api
        self.cfg = cfg
        self.det = False
        lens = cfg["lens"]
        q, k, v, do, cu_q, cu_k = inputs.varlen_inputs(lens, lens, cfg["Hq"], cfg["Hkv"], cfg["D"], cfg["dtype"],
                                                       seed=cfg["seed"], amp=cfg["amp"])
        self.host_in = (q, k, v, do)
        self.q, self.k, self.v, self.do = (t.to(dev) for t in (q, k, v, do))
        self.cu_q, self.cu_k = cu_q.to(dev), cu_k.to(dev)
        self.max_len = max(lens)
        self.out = torch.empty_like(self.q)
        self.lse = torch.empty(cfg["Hq"], q.shape[0], device=dev)
        self.dq, self.dk, self.dv = torch.empty_like(self.q), torch.empty_like(self.k), torch.empty_like(self.v)
        n = api.fa_bwd_varlen_workspace_size(len(lens), self.max_len, q.shape[0], cfg["Hq"], cfg["D"], False)
        self.ws = torch.empty(n, dtype=torch.uint8, device=dev)
        pairs = sum(visible_pairs(L, L, cfg["causal"], cfg["window"][0], cfg["window"][1]) for L in lens)
        self.flops_fwd = 4 * cfg["D"] * pairs * cfg["Hq"]
        self.flops_bwd = 10 * cfg["D"] * pairs * cfg["Hq"]
        self.kw = dict(scale=cfg["scale"], causal=cfg["causal"], window=cfg["window"], softcap=cfg["softcap"])

    def name(self):
        return "varlen%dxD%d" % (len(self.cfg["lens"]), self.cfg["D"])

    def run(self, tracer):
        api = self.api
        tracer.arm("fwd", self)
        api.fa_fwd_varlen(self.q, self.k, self.v, self.cu_q, self.cu_k, self.max_len, self.max_len, out=self.out,
                          lse=self.lse, **self.kw)
        n = api.fa_last_launch_count()
        tracer.arm("bwd", self)
        api.fa_bwd_varlen(self.do, self.q, self.k, self.v, self.out, self.lse, self.cu_q, self.cu_k, self.max_len,
                          self.max_len, self.dq, self.dk, self.dv, workspace=self.ws, **self.kw)
        tracer.disarm()
        return n + api.fa_last_launch_count()


class DecodeUnit:
    kind = "decode"

    def __init__(self, cfg, dev, num_splits=0, clean_l2=False):
        from exact_attention_121_b200 import api, inputs
        self.api = api
        self.cfg = cfg
        self.num_splits = num_splits
        # The first decode call of a step follows the backward kernels, whose
        # dirty L2 lines would otherwise be written back inside its span: a
        # 256 MB read (twice L2, outside the span, inside the step) writes
        # them back first and leaves clean lines.
        self.l2_buf = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=dev) if clean_l2 else None
        if clean_l2:
            self.l2_buf.fill_(0.0)
            self.l2_out = torch.empty((), dtype=torch.float32, device=dev)
        d = inputs.kvcache_inputs(cfg["B"], cfg["Hq"], cfg["Hkv"], cfg["D"], cfg["page_size"],
                                  cfg["pages_per_seq"], cfg["max_len"], Sq=1, Snew=1, dtype=cfg["dtype"],
                                  seed=cfg["seed"])
        self.host_in = (d["q"], d["k_new"], d["v_new"])
        self.q, self.kn, self.vn = (t.to(dev) for t in self.host_in)
        self.kc, self.vc = d["k_cache"].to(dev), d["v_cache"].to(dev)
        self.sl, self.bt = d["cache_seqlens"].to(dev), d["block_table"].to(dev)
        self.out = torch.empty_like(self.q)
        self.lse = torch.empty(cfg["B"], cfg["Hq"], 1, device=dev)
        self.rot = {}
        if cfg.get("rotary"):
            cos, sin = inputs.rotary_tables(cfg["max_len"] + 1, cfg["D"])
            self.rot = dict(rotary_cos=cos.to(dev), rotary_sin=sin.to(dev))
            n = api.fa_kvcache_rotary_workspace_size(cfg["B"], 1, cfg["Hq"], cfg["D"], num_splits)
        else:
            n = api.fa_kvcache_workspace_size(cfg["B"], 1, cfg["Hq"], cfg["D"], num_splits)
        self.ws = torch.empty(max(n, 256), dtype=torch.uint8, device=dev)
        lens = d["cache_seqlens"].numpy().astype(np.int64) + 1
        # algorithmic bytes: every attended K and V row once, plus q/out/new rows and the block table
        row = cfg["Hkv"] * cfg["D"] * 2
        self.bytes = int(2 * lens.sum() * row + 2 * self.q.numel() * 2 + 2 * self.kn.numel() * 2
                         + d["block_table"].numel() * 4 + lens.size * 4)
        self.flops_dec = int(4 * cfg["D"] * cfg["Hq"] * lens.sum())

    def name(self):
        base = "decode-rotary" if self.rot else "decode"
        return base + ("-s%d" % self.num_splits if self.num_splits > 0 else "")

    def run(self, tracer):
        if self.l2_buf is not None:
            torch.sum(self.l2_buf, dim=0, out=self.l2_out)
        tracer.arm("decode", self)
        self.api.fa_fwd_kvcache(self.q, self.kc, self.vc, self.kn, self.vn, self.sl, self.bt,
                                page_size=self.cfg["page_size"], out=self.out, lse=self.lse,
                                scale=self.cfg["scale"], causal=True, num_splits=self.num_splits,
                                workspace=self.ws, **self.rot)
        tracer.disarm()
        return self.api.fa_last_launch_count()

    def flops(self):
        return self.flops_dec

    def setup_e2e(self, pinned):
        self.pin_in = [pinned.get(t, i) for i, t in enumerate(self.host_in)]
        self.pin_out = [pinned.get_like(self.out)]

    def copy_in(self):
        for dst, src in zip((self.q, self.kn, self.vn), self.pin_in):
            dst.copy_(src, non_blocking=True)

    def copy_out(self):
        self.pin_out[0].copy_(self.out, non_blocking=True)

    def e2e_bytes(self):
        return (sum(t.numel() * t.element_size() for t in (self.q, self.kn, self.vn)),
                self.out.numel() * self.out.element_size())


class Fp8Unit:
    """FP8 (E4M3) forward through fa_fwd_fp8: q, k, v in, bf16 O out."""
    kind = "fp8"

    def __init__(self, cfg, dev):
        from exact_attention_121_b200 import api, inputs
        self.api = api
        self.cfg = cfg
        q, k, v, dq, dk, dv = inputs.fp8_inputs(cfg["B"], cfg["Sq"], cfg["Sk"], cfg["Hq"], cfg["Hkv"], cfg["D"],
                                                seed=cfg["seed"], amp=cfg["amp"])
        self.host_in = (q, k, v)
        self.q, self.k, self.v = (t.to(dev) for t in self.host_in)
        self.dq, self.dk, self.dv = (t.to(dev) for t in (dq, dk, dv))
        self.out = torch.empty(q.shape, dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty(cfg["B"], cfg["Hq"], cfg["Sq"], device=dev)
        self.flops_fwd8 = attn_flops(cfg)[0]
        self.kw = dict(scale=cfg["scale"], causal=cfg["causal"], window=cfg["window"], softcap=cfg["softcap"])

    def name(self):
        c = self.cfg
        return "fp8-H%dD%dS%d%s" % (c["Hq"], c["D"], c["Sq"], "c" if c["causal"] else "n")

    def run(self, tracer):
        tracer.arm("fwd8", self)
        self.api.fa_fwd_fp8(self.q, self.k, self.v, self.dq, self.dk, self.dv, out=self.out, lse=self.lse, **self.kw)
        tracer.disarm()
        return self.api.fa_last_launch_count()

    def flops(self):
        return self.flops_fwd8

    def setup_e2e(self, pinned):
        self.pin_in = [pinned.get(t, i) for i, t in enumerate(self.host_in)]
        self.pin_out = [pinned.get_like(self.out)]

    def copy_in(self):
        for dst, src in zip((self.q, self.k, self.v), self.pin_in):
            dst.copy_(src, non_blocking=True)

    def copy_out(self):
        self.pin_out[0].copy_(self.out, non_blocking=True)

    def e2e_bytes(self):
        return (sum(t.numel() * t.element_size() for t in (self.q, self.k, self.v)),
                self.out.numel() * self.out.element_size())


class Pinned:
    """Pinned host staging buffers: one per input tensor (each unit's own
    values), outputs shared between units of equal byte size (the copies out
    run in order on one stream)."""

    def __init__(self):
        self.pool = {}

    def _buf(self, nbytes, tag):
        key = (nbytes, tag)
        if key not in self.pool:
            self.pool[key] = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
        return self.pool[key]

    def get(self, t, slot):
        view = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
        view.copy_(t)
        return view

    def get_like(self, t):
        nb = t.numel() * t.element_size()
        return self._buf(nb, "out%d" % nb).view(t.dtype).view(t.shape)


class Tracer:
    """Two kinds of CUDA event pairs, accumulated per kernel class over the
    timed region: one immediately around each call's dominant kernel (set
    through fa_set_trace_events, recorded by the library on the launching
    stream), and one around the whole API call (every kernel of the call,
    recorded on the same stream).  A call span runs from arm() to the next
    arm() or disarm()."""

    def __init__(self, lib, enabled=False, kernel_classes=("fwd", "bwd", "fwd8", "decode")):
        self.lib = lib
        self.enabled = enabled
        # classes whose dominant kernel gets its own event pair; the others
        # get the call span only (an event recorded between the decode split
        # kernel and its dependent combine kernel would serialise them)
        self.kernel_classes = kernel_classes
        self.pending = []
        self.pending_calls = []
        self.totals = {}
        self.per_unit = {}
        self.per_call = {}
        self._open = None

    def _work(self, cls, unit):
        return {"fwd": getattr(unit, "flops_fwd", 0), "bwd": getattr(unit, "flops_bwd", 0),
                "fwd8": getattr(unit, "flops_fwd8", 0), "decode": getattr(unit, "bytes", 0)}[cls]

    def _close_call(self):
        if self._open is not None:
            cls, name, a, work = self._open
            b = torch.cuda.Event(enable_timing=True)
            b.record()
            self.pending_calls.append((cls, name, a, b, work))
            self._open = None

    def arm(self, cls, unit):
        if not self.enabled:
            return
        self._close_call()
        work = self._work(cls, unit)
        c = torch.cuda.Event(enable_timing=True)
        c.record()
        self._open = (cls, unit.name(), c, work)
        if cls not in self.kernel_classes:
            return
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        b.record()
        self.lib.fa_set_trace_events(a.cuda_event, b.cuda_event)
        self.pending.append((cls, unit.name(), a, b, work))

    def disarm(self):
        if self.enabled:
            self.lib.fa_set_trace_events(None, None)
            self._close_call()

    def collect(self):
        """Totals per kernel class; per (class, unit) kernel totals in
        self.per_unit and whole-call totals in self.per_call, each
        [ms, count, work]."""
        for cls, name, a, b, work in self.pending:
            ms = a.elapsed_time(b)
            for d, key in ((self.totals, cls), (self.per_unit, (cls, name))):
                t = d.setdefault(key, [0.0, 0, 0])
                t[0] += ms
                t[1] += 1
                t[2] += work
        for cls, name, a, b, work in self.pending_calls:
            t = self.per_call.setdefault((cls, name), [0.0, 0, 0])
            t[0] += a.elapsed_time(b)
            t[1] += 1
            t[2] += work
        self.pending = []
        self.pending_calls = []
        return self.totals


# ---------------------------------------------------------------------------
# arms
# ---------------------------------------------------------------------------

def build_units(dev, workload, point=None):
    from exact_attention_121_b200 import inputs
    units = []
    if workload in ("full", "sweep", "point"):
        for cfg in inputs.seqlen_sweep_configs():
            u_name = "H%dD%dS%d%s" % (cfg["Hq"], cfg["D"], cfg["Sq"], "c" if cfg["causal"] else "n")
            if workload == "point" and u_name != point:
                continue
            units.append(AttnUnit(cfg, dev))
    if workload in ("full", "gqa"):
        units.append(AttnUnit(inputs.gqa_local_config(), dev))
        units.append(AttnUnit(inputs.gqa_local_config(), dev, deterministic=True))
    if workload in ("full", "decode"):
        units.append(DecodeUnit(inputs.paged_decode_config(), dev, clean_l2=(workload == "full")))
        for n in (1, 4, 16):
            units.append(DecodeUnit(inputs.paged_decode_config(), dev, num_splits=n))
    if workload == "small":
        units.append(AttnUnit(inputs.fwd_bwd_512_config(), dev))
    if workload == "varlen":
        units.append(VarlenUnit(inputs.varlen_config(), dev))
    if workload == "decode_rotary":
        units.append(DecodeUnit(inputs.paged_decode_rotary_config(), dev))
    if workload == "fp8":
        units.append(Fp8Unit(inputs.fp8_config(), dev))
    if workload == "alibi":
        units.append(AttnUnit(inputs.alibi_config(), dev))
    return units


def time_steps(units, steps, warmup, tracer, e2e=False, barrier=None):
    """Device time of `steps` steps.  With e2e, every unit's inputs come from
    pinned host memory on a copy-in stream and its outputs go back on a
    copy-out stream, overlapped with the other units' kernels: unit u's
    kernels wait for its inputs, its copy-out waits for its kernels, its next
    copy-in waits for its kernels and its next kernels wait for its copy-out."""
    stream = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    launches = 0

    def one_step(tr, ev):
        n = 0
        for i, u in enumerate(units):
            if not e2e:
                n += u.run(tr)
                continue
            with torch.cuda.stream(s_in):
                if ev["done"][i] is not None:
                    s_in.wait_event(ev["done"][i])
                u.copy_in()
                e_in = torch.cuda.Event()
                e_in.record(s_in)
            stream.wait_event(e_in)
            if ev["out"][i] is not None:
                stream.wait_event(ev["out"][i])
            n += u.run(tr)
            e_done = torch.cuda.Event()
            e_done.record(stream)
            ev["done"][i] = e_done
            with torch.cuda.stream(s_out):
                s_out.wait_event(e_done)
                u.copy_out()
                e_out = torch.cuda.Event()
                e_out.record(s_out)
            ev["out"][i] = e_out
        return n

    ev = {"done": [None] * len(units), "out": [None] * len(units)}
    for _ in range(warmup):
        one_step(Tracer(tracer.lib), ev)
    torch.cuda.synchronize()
    if barrier:
        barrier()
    torch.cuda.synchronize()
    ev = {"done": [None] * len(units), "out": [None] * len(units)}
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    s_in.wait_event(start)
    s_out.wait_event(start)
    for _ in range(steps):
        launches += one_step(tracer, ev)
    # the step ends when the last result is back in host memory
    for side in (s_in, s_out):
        e_end = torch.cuda.Event()
        e_end.record(side)
        stream.wait_event(e_end)
    stop.record(stream)
    torch.cuda.synchronize()
    if barrier:
        barrier()
    return start.elapsed_time(stop), launches


def cpu_oracle_sample(budget_s=12.0):
    """Time the float64 oracle on head slices of the seqlen-sweep point S=2048,
    D=128 (forward + backward) for about budget_s seconds; TFLOP/s."""
    import oracle
    from exact_attention_121_b200 import inputs
    cfg = next(c for c in inputs.seqlen_sweep_configs() if c["Sq"] == 2048 and c["D"] == 128 and c["causal"])
    q, k, v, do = inputs.attention_inputs(cfg["B"], cfg["Sq"], cfg["Sk"], cfg["Hq"], cfg["Hkv"], cfg["D"],
                                          cfg["dtype"], seed=cfg["seed"])
    f = lambda t, b, h: t[b:b + 1, :, h:h + 1].double().numpy()
    one = dict(cfg, B=1, Hq=1, Hkv=1)
    flops = sum(attn_flops(one))
    t0 = time.perf_counter()
    n = 0
    while True:
        b, h = n % cfg["B"], (n // cfg["B"]) % cfg["Hq"]
        oracle.attn_fwd(f(q, b, h), f(k, b, h), f(v, b, h), cfg["scale"], cfg["causal"])
        oracle.attn_bwd(f(do, b, h), f(q, b, h), f(k, b, h), f(v, b, h), cfg["scale"], cfg["causal"])
        n += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    try:
        from threadpoolctl import threadpool_info
        cores = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:  # noqa: BLE001
        cores = os.cpu_count()
    return dict(value=n * flops / el / 1e12, unit="TFLOP/s", cores=int(cores), kind="oracle",
                sample=f"{n} (batch, head) slices of the S=2048 D=128 causal sweep point, fwd+bwd in float64, "
                       f"{el:.1f} s", elapsed_s=el, flops=n * flops)


def _r(x, n=4):
    return float(f"{x:.{n}g}")


def per_config(tracer, peaks):
    """Per workload point, from the whole-call event spans of the timed
    region: forward and forward+backward TFLOP/s of every attention point
    and their fractions of the measured bf16 tensor rates (sustained and
    burst); GB/s of every paged-decode call (append + split-KV attention +
    combine) beside its split kernel's, as fractions of the measured HBM
    copy bandwidth."""
    sus, burst, hbm = peaks["bf16_tflops_sustained"], peaks["bf16_tflops"], peaks["hbm_gbs"]
    out = {}
    for name in sorted({n for (_, n) in tracer.per_call}):
        e = {}
        f = tracer.per_call.get(("fwd", name)) or tracer.per_call.get(("fwd8", name))
        bw = tracer.per_call.get(("bwd", name))
        dc = tracer.per_call.get(("decode", name))
        if f:
            peak_scale = FP8_OVER_BF16 if ("fwd8", name) in tracer.per_call else 1.0
            ms_f = f[0] / f[1]
            tf = f[2] / f[1] / (ms_f / 1e3) / 1e12
            e.update(fwd_ms=_r(ms_f), fwd_tflops=_r(tf), fwd_frac=_r(tf / (sus * peak_scale), 3),
                     fwd_frac_burst=_r(tf / (burst * peak_scale), 3))
        if f and bw:
            ms_b = bw[0] / bw[1]
            tb = bw[2] / bw[1] / (ms_b / 1e3) / 1e12
            tfb = (f[2] / f[1] + bw[2] / bw[1]) / ((ms_f + ms_b) / 1e3) / 1e12
            e.update(bwd_ms=_r(ms_b), bwd_tflops=_r(tb), fwdbwd_tflops=_r(tfb), fwdbwd_frac=_r(tfb / sus, 3),
                     fwdbwd_frac_burst=_r(tfb / burst, 3))
        if dc:
            ms = dc[0] / dc[1]
            gbs = dc[2] / dc[1] / (ms / 1e3) / 1e9
            e.update(call_ms=_r(ms), call_gbs=_r(gbs), call_frac=_r(gbs / hbm, 3))
            kt = tracer.per_unit.get(("decode", name))
            if kt:
                kg = kt[2] / kt[1] / (kt[0] / kt[1] / 1e3) / 1e9
                e.update(split_kernel_gbs=_r(kg), split_kernel_frac=_r(kg / hbm, 3))
        out[name] = e
    # the long-sequence head-dim-128 sweep points (S >= 4096), both masks
    long128 = [v for n, v in out.items() if n.startswith("H16D128S") and "-" not in n
               and int(n[8:-1]) >= 4096 and "fwd_frac" in v]
    summary = {}
    if long128:
        summary["d128_s4k_plus"] = {"fwd_frac_min": min(v["fwd_frac"] for v in long128),
                                    "fwdbwd_frac_min": min(v["fwdbwd_frac"] for v in long128 if "fwdbwd_frac" in v),
                                    "points": len(long128)}
    dec = [v["call_frac"] for n, v in out.items() if n.startswith("decode") and "call_frac" in v]
    if dec:
        summary["decode_call_frac_min"] = min(dec)
    return out, summary


def max_over_ranks(ms, pg, dev):
    """The slowest rank's time: every rank contributes its own device-timed
    milliseconds (one all-reduce, taken in the same order on every rank)."""
    if pg is None:
        return float(ms)
    t = torch.tensor([float(ms)], dtype=torch.float64, device=dev)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(world, flops_step, steps, ms):
    """Aggregate throughput of `world` replicas, each of which ran `steps`
    steps of `flops_step` flops, over the slowest rank's `ms`."""
    return world * flops_step * steps / (ms / 1e3) / 1e12


def reference_arm(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    for _ in range(args.warmup):
        cpu_oracle_sample(budget_s=0.0)
    samples = [cpu_oracle_sample(budget_s=0.0) for _ in range(args.steps)]
    total_s = sum(s["elapsed_s"] for s in samples)
    value = sum(s["flops"] for s in samples) / total_s / 1e12
    cb = {k: samples[0][k] for k in ("unit", "cores", "kind")}
    cb["value"] = value
    cb["sample"] = f"each step: one (batch, head) slice of the S=2048 D=128 causal sweep point, fwd+bwd in float64"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * total_s / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": "oracle on sampled slices of the step's workload"},
            "cpu_baseline": cb,
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="full", choices=["full", "sweep", "gqa", "decode", "small", "point", "varlen",
                                                                   "alibi", "decode_rotary", "fp8"])
    ap.add_argument("--point", default="H16D128S4096n", help="sweep point for --workload point")
    ap.add_argument("--e2e-steps", type=int, default=2)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--detail", action="store_true", help="also print per-unit times")
    args = ap.parse_args()
    if args.impl == "reference":
        return reference_arm(args)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
        pg = dist

    def barrier():
        if pg:
            pg.barrier()

    from exact_attention_121_b200 import _lib
    lib = _lib.load()
    units = build_units(dev, args.workload, args.point)
    flops_step = sum(u.flops() for u in units)
    peaks, peak_src = load_peaks()

    # device-resident timing with per-call events and, except for decode,
    # per-kernel trace events
    tracer = Tracer(lib, enabled=True, kernel_classes=("fwd", "bwd", "fwd8"))
    gidx = os.environ.get("CUDA_VISIBLE_DEVICES", str(local)).split(",")[local] if "CUDA_VISIBLE_DEVICES" in os.environ else str(local)
    clocks = ClockSampler(gidx)
    clocks.start()
    ms, launches = time_steps(units, args.steps, args.warmup, tracer, barrier=barrier)
    clk = clocks.stop()
    totals = tracer.collect()
    dec_units = [u for u in units if u.kind == "decode"]
    if dec_units:
        # the decode split kernel alone, in a short separate pass
        ktr = Tracer(lib, enabled=True)
        time_steps(dec_units, 3, 1, ktr)
        for cls, v in ktr.collect().items():
            totals[cls] = v
        tracer.per_unit.update({k: v for k, v in ktr.per_unit.items() if k[0] == "decode"})
    points, points_summary = per_config(tracer, peaks)
    ms_max = max_over_ranks(ms, pg, dev)
    value = whole_job_tflops(world, flops_step, args.steps, ms_max)

    # per-unit detail (untimed for the headline; separate short pass)
    detail = {}
    if args.detail and rank == 0:
        for u in units:
            tr = Tracer(lib, enabled=True)
            t_ms, _ = time_steps([u], 3, 1, tr)
            tt = tr.collect()
            d = {"ms": t_ms / 3, "tflops": u.flops() / (t_ms / 3 / 1e3) / 1e12}
            for cls, (kms, cnt, work) in tt.items():
                d[cls + "_ms"] = kms / cnt
                d[cls + ("_gbs" if cls == "decode" else "_tflops")] = (work / cnt) / (kms / cnt / 1e3) / (1e9 if cls == "decode" else 1e12)
            detail[u.name()] = d

    # end to end through the C ABI with pinned host buffers
    pinned = Pinned()
    for u in units:
        u.setup_e2e(pinned)
    h2d = sum(u.e2e_bytes()[0] for u in units)
    d2h = sum(u.e2e_bytes()[1] for u in units)
    ms_e2e, _ = time_steps(units, args.e2e_steps, 1, Tracer(lib), e2e=True, barrier=barrier)
    ms_e2e = max_over_ranks(ms_e2e, pg, dev)
    e2e_value = whole_job_tflops(world, flops_step, args.e2e_steps, ms_e2e)

    # Roofline of the dominant kernel class (largest traced time), per launch
    # of the representative sweep point when it ran (so that `achieved` and
    # the ncu `traffic` describe the same launch), else over all its launches.
    dom = max(totals.items(), key=lambda kv: kv[1][0])
    cls, (kms_all, cnt_all, work_all) = dom
    rep = ROOFLINE_UNIT[cls]
    kms, cnt, work = tracer.per_unit.get((cls, rep), (kms_all, cnt_all, work_all))
    if (cls, rep) not in tracer.per_unit:
        rep = "all launches"
    scale = 1e9 if cls == "decode" else 1e12
    achieved = (work / cnt) / (kms / cnt / 1e3) / scale
    achieved_all = work_all / (kms_all / 1e3) / scale
    if cls == "decode":
        pk = peaks["hbm_gbs"]
        roof = {"bound": "hbm", "achieved": achieved, "peak": pk, "unit": "GB/s", "frac": achieved / pk}
    elif cls == "fwd8":
        pk = peaks["bf16_tflops_sustained"] * FP8_OVER_BF16
        roof = {"bound": "tensor", "achieved": achieved, "peak": pk, "unit": "TFLOP/s", "frac": achieved / pk}
    else:
        pk = peaks["bf16_tflops_sustained"]
        roof = {"bound": "tensor", "achieved": achieved, "peak": pk, "unit": "TFLOP/s", "frac": achieved / pk}
    if cls != "decode":
        # exponentials: one per visible (query, key) pair in either pass, i.e.
        # flops / (4 D) forward, flops / (10 D) backward, head dim 128 here;
        # nominal MUFU rate 16 per clock per SM at the sampled SM clock
        exps = (work / cnt) / ((10 if cls == "bwd" else 4) * 128)
        exp_rate = exps / (kms / cnt / 1e3)
        exp_peak = 16 * 148 * ((clk or {}).get("sm_mhz") or 1965.0) * 1e6
        roof["sfu"] = {"exp_per_launch": exps, "exp_per_s": exp_rate, "peak_exp_per_s": exp_peak,
                       "frac": exp_rate / exp_peak, "peak_source": "nominal 16/clk/SM x 148 SMs x sampled SM clock"}
    roof["traffic"] = TRAFFIC_PER_LAUNCH.get((cls, rep))
    roof["launch"] = rep
    roof["algorithmic_per_launch"] = work / cnt
    roof["achieved_all_launches"] = achieved_all
    roof["kernel"] = {"fwd": "fwd_tc_kernel (tcgen05 forward)", "bwd": "bwd_tc_kernel (tcgen05 backward)",
                      "fwd8": "fwd_tc_kernel<E4M3> (tcgen05 kind::f8f6f4 forward)",
                      "decode": "decode_tma_kernel (split-KV decode)"}[cls]
    roof["peak_source"] = f"{peak_src} " + {"decode": "(hbm_gbs)", "fwd8": "(bf16_tflops_sustained x 2, e4m3/bf16 "
                                                       "nominal ratio)"}.get(cls, "(bf16_tflops_sustained)")
    kernels = {c: {"ms_total": v[0], "launches": v[1],
                   ("gbs" if c == "decode" else "tflops"): v[2] / (v[0] / 1e3) / (1e9 if c == "decode" else 1e12)}
               for c, v in totals.items()}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_oracle_sample()

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "e4m3" if args.workload == "fp8" else "bf16",
                "data": "synthetic",
                "config": {"workload": args.workload + ": " + ", ".join(u.name() for u in units),
                           "l2": "inputs larger than L2 (no flush)" + (
                               "; a 256 MB read before the first decode call" if args.workload == "full" else ""),
                           "parallelism": f"replicas x{world}",
                           "flops_per_step": flops_step},
                "gpu_launches": launches,
                "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                        "d2h_bytes_per_step": d2h, "steps": args.e2e_steps},
                "roofline": roof, "kernels": kernels, "per_config": points, "per_config_summary": points_summary,
                "peaks": {"source": peak_src, "bf16_tflops_sustained": peaks["bf16_tflops_sustained"],
                          "bf16_tflops": peaks["bf16_tflops"], "hbm_gbs": peaks["hbm_gbs"]},
                "cpu_baseline": cpu, "clocks": clk}
        if detail:
            line["detail"] = detail
        print(json.dumps(line))
    if pg:
        pg.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
