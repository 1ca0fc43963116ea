#!/usr/bin/env python3
"""Throughput of the shared-prefix attention + candidate readout hot path.

One step = one jev_prefix_suffix_attn (one attention layer, all heads, all
branches) + one jev_candidate_readout over one batch of synthetic input (the
tree workload: jev_tree_attn + readout).  The headline metric is suffix
tokens/s.  Steps are replayed from CUDA graphs over rotating copies of the
inputs whose total size exceeds twice the L2, so every step reads its prefix
cache and suffix tensors from HBM.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload wide_7b] [--impl jev|reference]

With N > 1 (torchrun) every rank runs an independent replica of the workload
on its own GPU (no collective on the data path; weak scaling); the step time
is the max over ranks.  --impl reference times the fp64 CPU oracle on the
host cores instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "suffix tokens/s (shared-prefix attn + readout) and % of roofline, 1 B200"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def _peak_number(v):
    """A peak figure as a float: a plain number, or a record holding one under
    "value", "median" or "mean"; None otherwise."""
    if isinstance(v, bool):
        return None
    if isinstance(v, (int, float)):
        return float(v) if v > 0 else None
    if isinstance(v, dict):
        for k in ("value", "median", "mean"):
            if k in v:
                return _peak_number(v[k])
    return None


def peaks(path=None):
    """Roofline denominators: the measured HBM copy bandwidth (GB/s) and bf16
    GEMM throughput (TFLOP/s, burst and sustained) of this machine's B200s
    from MEASURED_PEAKS.json at the repository root, each figure found at the
    top level or one object down; any figure the file lacks (or no file) takes
    the fallback value, and the source says which."""
    p = path or os.path.join(ROOT, "MEASURED_PEAKS.json")
    d = {}
    if os.path.exists(p):
        try:
            with open(p) as f:
                d = json.load(f)
        except (OSError, ValueError):
            d = {}
    if not isinstance(d, dict):
        d = {}
    out, found = dict(FALLBACK_PEAKS), []
    for key in FALLBACK_PEAKS:
        v = _peak_number(d.get(key))
        if v is None:
            for sub in d.values():
                if isinstance(sub, dict) and _peak_number(sub.get(key)) is not None:
                    v = _peak_number(sub.get(key))
                    break
        if v is not None:
            out[key] = v
            found.append(key)
    if len(found) == len(FALLBACK_PEAKS):
        return out, "measured"
    if found:
        return out, "measured (" + ", ".join(found) + "), fallback for the rest"
    return out, "fallback"


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


# ----------------------------------------------------------------------------- algorithmic work


def flat_work(c) -> dict:
    """Algorithmic FLOPs and unique bytes of one step (prefix K/V counted once)."""
    cfg = c.cfg
    s = 2 if cfg.dtype == synth.BF16 else 4
    Ls = np.diff(c.cu_seqlens).astype(np.int64)
    T = int(Ls.sum())
    f_attn = 4 * T * cfg.Hq * cfg.Lp * cfg.d + 4 * cfg.Hq * cfg.d * int((Ls * (Ls + 1) // 2).sum())
    n_pairs = int(c.pair_tok.size)
    f_read = 2 * cfg.H * n_pairs
    b_attn = s * (2 * T * cfg.Hq * cfg.d + 2 * cfg.Lp * cfg.Hkv * cfg.d + 2 * T * cfg.Hkv * cfg.d) + 4 * T * cfg.Hq
    b_read = s * (cfg.B * cfg.H + n_pairs * cfg.H) + 8 * n_pairs + 4 * cfg.B
    return dict(T=T, B=cfg.B, flops_attn=f_attn, flops_readout=f_read, bytes_attn=b_attn, bytes_readout=b_read)


# ----------------------------------------------------------------------------- clocks


class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap,utilization.gpu")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"jev_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                p = [x.strip() for x in line.split(",")]
                if len(p) >= 10:
                    rows.append(p)
        os.remove(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        loaded = [r for r in rows if (num(r[9]) or 0) > 0] or rows
        sm = [num(r[1]) for r in loaded if num(r[1]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in loaded for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": num(rows[0][2]),
                "reasons": reasons, "samples": len(rows), "samples_under_load": len(loaded),
                "power_w_max": max((num(r[3]) or 0) for r in rows)}


# ----------------------------------------------------------------------------- reference arm (oracle on CPU)


class OracleSampler:
    """Times the fp64 oracle on bounded samples of a flat workload and scales
    the sample times to the whole workload: attention is sampled by (token,
    head) rows, the readout (full-vocabulary logits + log-softmax) by option
    sets.  Workload time = rows * (time per sampled row) + sets * (time per
    sampled set); tokens/s = suffix tokens / workload time."""

    def __init__(self, cfg):
        import oracle
        self.oracle = oracle
        self.cfg = cfg
        self.c = synth.flat_case(cfg, with_lm_head=False)
        self.W = synth.lm_head(cfg.seed, cfg.V, cfg.H, cfg.dtype, cfg.w_std)
        self.T = self.c.T
        self.rng = np.random.default_rng(1234)
        self.t_rows = self.n_rows = 0
        self.t_sets = self.n_sets = 0
        self.cost_row = self._attn(16)[0] / 16
        self.cost_set = self._readout(1)[0]
        self.reset()

    def reset(self):
        """Forget the sampled times so far (after warm-up)."""
        self.t_rows = self.n_rows = self.t_sets = self.n_sets = 0

    def _attn(self, n):
        c = self.c
        rows = np.stack([self.rng.integers(0, self.T, n), self.rng.integers(0, self.cfg.Hq, n)], 1).astype(np.int32)
        t0 = time.perf_counter()
        self.oracle.prefix_suffix_attn(c.q, c.k_pre, c.v_pre, c.k_suf, c.v_suf, c.cu_seqlens, theta=self.cfg.theta,
                                       rows=rows)
        dt = time.perf_counter() - t0
        self.t_rows += dt
        self.n_rows += n
        return dt, n

    def _readout(self, n):
        c = self.c
        s0 = int(self.rng.integers(0, self.cfg.B - n + 1))
        so = c.set_offsets[s0:s0 + n + 1] - c.set_offsets[s0]
        toks = c.pair_tok[c.set_offsets[s0]:c.set_offsets[s0 + n]]
        t0 = time.perf_counter()
        self.oracle.candidate_readout(c.hidden[s0:s0 + n], self.W, so, toks, full_vocab=True)
        dt = time.perf_counter() - t0
        self.t_sets += dt
        self.n_sets += n
        return dt, n

    def step(self, budget_s):
        """One sample costing about budget_s: attention rows and readout sets
        in proportion to their share of the whole workload's oracle time."""
        full_attn = self.cost_row * self.T * self.cfg.Hq
        full_read = self.cost_set * self.cfg.B
        f_attn = full_attn / (full_attn + full_read)
        n_rows = int(max(1, min(self.T * self.cfg.Hq, f_attn * budget_s / self.cost_row)))
        self._attn(n_rows)
        n_sets = int(min(self.cfg.B, (1 - f_attn) * budget_s / self.cost_set))
        if n_sets >= 1 or self.n_sets == 0:
            self._readout(max(1, n_sets))

    def tokens_per_s(self):
        t = (self.t_rows / self.n_rows) * self.T * self.cfg.Hq + (self.t_sets / self.n_sets) * self.cfg.B
        return self.T / t

    def describe(self):
        return (f"{self.n_rows} (token, head) attention rows and {self.n_sets} option sets (full-vocabulary logits) "
                f"of the workload ({self.T} tokens x {self.cfg.Hq} heads, {self.cfg.B} sets), {self.t_rows + self.t_sets:.1f} s "
                f"of oracle time, scaled to the whole workload")


class TreeOracleSampler:
    """Times the fp64 oracle on bounded samples of the tree workload and
    scales them to the whole workload.  Attention is sampled by question: one
    question's subtree (its tokens and all its option leaves over the root
    cache) is an independent tree problem, so its oracle time over its unique
    tokens gives a time per tree token.  The readout is sampled by option set
    (one question's leaves, full-vocabulary logits of every used row).
    Workload time = N * (time per sampled token) + sets * (time per sampled
    set); tokens/s = N / workload time."""

    def __init__(self, cfg):
        import oracle
        self.oracle = oracle
        self.cfg = cfg
        self.tc = tc = synth.tree_case(cfg, with_lm_head=False)
        self.W = synth.lm_head(cfg.seed, cfg.V, cfg.H, cfg.dtype, cfg.w_std)
        self.trie = oracle.trie_build(tc.seq_off, tc.toks, cfg.Lp)
        self.T = int(self.trie["tok_off"][-1])
        self.n_sets = tc.set_offsets.size - 1
        self.co, self.prow, self.tix = oracle.tree_readout_pairs(tc.seq_off, tc.score_from, self.trie["path_row"],
                                                                 tc.set_offsets)
        self.rng = np.random.default_rng(1234)
        self.t_tok = self.n_tok = self.t_sets = self.n_sets_done = 0
        self.cost_tok = self._attn()[0] / max(1, self.n_tok)
        self.cost_set = self._readout()[0]
        self.reset()

    def reset(self):
        """Forget the sampled times so far (after warm-up)."""
        self.t_tok = self.n_tok = self.t_sets = self.n_sets_done = 0

    def _attn(self):
        tc, cfg = self.tc, self.cfg
        qi = int(self.rng.integers(0, self.n_sets))
        c0, c1 = int(tc.set_offsets[qi]), int(tc.set_offsets[qi + 1])
        so = (tc.seq_off[c0:c1 + 1] - tc.seq_off[c0]).astype(np.int32)
        toks = tc.toks[tc.seq_off[c0]:tc.seq_off[c1]]
        sub = self.oracle.trie_build(so, toks, cfg.Lp)
        n = int(sub["tok_off"][-1])
        gather = np.zeros(n, np.int64)
        gather[sub["path_row"]] = self.trie["path_row"][tc.seq_off[c0]:tc.seq_off[c1]]
        q, k, v = tc.q[gather], tc.k[gather], tc.v[gather]
        t0 = time.perf_counter()
        self.oracle.tree_attn(sub, q, k, v, tc.k_root, tc.v_root, theta=cfg.theta)
        dt = time.perf_counter() - t0
        self.t_tok += dt
        self.n_tok += n
        return dt, n

    def _readout(self):
        tc = self.tc
        qi = int(self.rng.integers(0, self.n_sets))
        c0, c1 = int(tc.set_offsets[qi]), int(tc.set_offsets[qi + 1])
        p0, p1 = int(self.co[c0]), int(self.co[c1])
        co = (self.co[c0:c1 + 1] - p0).astype(np.int32)
        t0 = time.perf_counter()
        self.oracle.candidate_readout(tc.hidden, self.W, np.array([0, c1 - c0], np.int32),
                                      tc.toks[self.tix[p0:p1]], cand_offsets=co, pair_row=self.prow[p0:p1],
                                      full_vocab=True)
        dt = time.perf_counter() - t0
        self.t_sets += dt
        self.n_sets_done += 1
        return dt, 1

    def step(self, budget_s):
        full_attn = self.cost_tok * self.T
        full_read = self.cost_set * self.n_sets
        f_attn = full_attn / (full_attn + full_read)
        spent = 0.0
        while spent < f_attn * budget_s or self.n_tok == 0:
            spent += self._attn()[0]
        spent = 0.0
        while spent < (1 - f_attn) * budget_s or self.n_sets_done == 0:
            spent += self._readout()[0]

    def tokens_per_s(self):
        t = (self.t_tok / self.n_tok) * self.T + (self.t_sets / self.n_sets_done) * self.n_sets
        return self.T / t

    def describe(self):
        return (f"{self.n_tok} tree tokens of question subtrees (all heads, root {self.cfg.Lp} keys) and "
                f"{self.n_sets_done} option sets (full-vocabulary logits) of the workload ({self.T} tree tokens, "
                f"{self.n_sets} sets), {self.t_tok + self.t_sets:.1f} s of oracle time, scaled to the whole workload")


def make_sampler(cfg):
    return TreeOracleSampler(cfg) if isinstance(cfg, synth.TreeConfig) else OracleSampler(cfg)


def workload_tokens(cfg) -> tuple:
    """(suffix or tree tokens, branches or candidates) of a workload, from the generator alone."""
    if isinstance(cfg, synth.TreeConfig):
        tc = synth.tree_case(cfg, with_lm_head=False)
        return int(tc.n_unique), int(tc.seq_off.size - 1)
    return int(synth.suffix_lengths(cfg).sum()), cfg.B


L2_NOTE = "per-step inputs rotate over device copies totalling more than twice the 126 MB L2"


def bench_config(wl_name: str, world: int, T: int, B: int) -> dict:
    """The workload description both arms print (identical keys and values)."""
    cfg = synth.CONFIGS[wl_name]
    return {"workload": synth.WORKLOAD_TEXT[wl_name], "global_batch": B * world, "seq_len": cfg.Lp,
            "suffix_tokens_per_replica": T, "parallelism": f"replicas{world}" if world > 1 else "single",
            "l2": L2_NOTE}


def reference_arm(args, wl_name):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    cfg = synth.CONFIGS[wl_name]
    total_budget = float(os.environ.get("JEV_REF_TOTAL_S", "120"))
    per_step = max(0.002, total_budget / (args.steps + args.warmup))
    smp = make_sampler(cfg)
    for _ in range(args.warmup):
        smp.step(per_step)
    smp.reset()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        smp.step(per_step)
    wall = time.perf_counter() - t0
    value = smp.tokens_per_s()
    cores = host_cores()
    T, B = workload_tokens(cfg)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * wall / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": bench_config(wl_name, world, T, B),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": "all timed steps together: " + smp.describe()},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


def cpu_baseline(cfg, budget_s: float) -> dict:
    """The oracle timed on bounded samples of the workload for about budget_s seconds."""
    smp = make_sampler(cfg)
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < budget_s:
        smp.step(min(2.0, budget_s / 4))
    return {"value": smp.tokens_per_s(), "unit": "tokens/s", "cores": host_cores(), "kind": "oracle",
            "sample": smp.describe()}


# ----------------------------------------------------------------------------- jev arm


def traffic_of(kernel: str, workload: str, src_files):
    """DRAM traffic per launch from a committed ncu summary, if the kernel's
    sources have not changed since it was taken (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(f"{kernel}/{workload}")
    if not e:
        return None
    h = hashlib.sha256()
    for fn in src_files:
        with open(os.path.join(ROOT, fn), "rb") as f:
            h.update(f.read())
    return e["bytes_per_launch"] if e.get("src_sha256") == h.hexdigest() else None


KERNEL_SRC = {
    "attn_tc": ["attention_cascade_b200/csrc/attn_tc.cu", "attention_cascade_b200/csrc/attn_tc1.cu",
                "attention_cascade_b200/csrc/attn_tc_common.cuh", "attention_cascade_b200/csrc/common.cuh",
                "attention_cascade_b200/csrc/tc_ptx.cuh", "attention_cascade_b200/csrc/kernels.h"],
    "attn_simt": ["attention_cascade_b200/csrc/attn_simt.cu", "attention_cascade_b200/csrc/common.cuh"],
}


class FlatWorkload:
    """Shared-prefix attention (one layer, all heads, all branches) + readout."""

    def __init__(self, cfg, dev, jev, torch):
        self.cfg, self.jev, self.torch = cfg, jev, torch
        c = synth.flat_case(cfg, with_lm_head=False)
        self.c = c
        self.work = flat_work(c)
        self.T, self.B = self.work["T"], cfg.B
        self.tdt = torch.bfloat16 if cfg.dtype == synth.BF16 else torch.float32
        self.W = load_lm_head(cfg, dev, torch, self.tdt)
        self.base = dict(q=to_dev(c.q, dev, torch), k_pre=to_dev(c.k_pre, dev, torch), v_pre=to_dev(c.v_pre, dev, torch),
                         k_suf=to_dev(c.k_suf, dev, torch), v_suf=to_dev(c.v_suf, dev, torch),
                         hidden=to_dev(c.hidden, dev, torch), pair_tok=to_dev(c.pair_tok, dev, torch))
        self.cu = to_dev(c.cu_seqlens, dev, torch)
        self.so = to_dev(c.set_offsets, dev, torch)
        desc = jev.make_attn_desc(cfg.B, cfg.Lp, cfg.Hq, cfg.Hkv, cfg.d, self.T,
                                  jev.JEV_BF16 if self.tdt == torch.bfloat16 else jev.JEV_F32, cfg.theta)
        self.ws = jev.new_workspace(jev.jev_prefix_suffix_attn_workspace(desc), dev)
        self.out = torch.empty_like(self.base["q"])
        self.lse = torch.empty((self.T, cfg.Hq), dtype=torch.float32, device=dev)
        self.lp = torch.empty(c.pair_tok.size, dtype=torch.float32, device=dev)
        self.choice = torch.empty(cfg.B, dtype=torch.int32, device=dev)
        self.e2e_inputs = ("q", "k_suf", "v_suf", "hidden", "pair_tok")

    def attn(self, cp, s):
        self.jev.jev_prefix_suffix_attn(cp["q"], cp["k_pre"], cp["v_pre"], cp["k_suf"], cp["v_suf"], cp.get("cu", self.cu),
                                        out=self.out, lse=self.lse, workspace=self.ws, rope_theta=self.cfg.theta, stream=s)

    def readout(self, cp, s):
        self.jev.jev_candidate_readout(cp["hidden"], self.W, cp.get("so", self.so), cp["pair_tok"], logprob=self.lp,
                                       choice=self.choice, stream=s)

    def e2e_host(self):
        """Host-side inputs of one request (pinned) and the per-step host work."""
        t = self.torch
        h = {k: self.base[k].cpu().pin_memory() for k in self.e2e_inputs}
        h["cu"] = self.cu.cpu().pin_memory()
        h["so"] = self.so.cpu().pin_memory()
        return h

    def host_prep(self, h):
        return h

    def describe_e2e(self):
        return ("per step: one pinned H2D copy of a staging buffer holding suffix q/k/v, cu_seqlens, hidden rows "
                "and option sets; both API calls; one D2H copy of log-probs and choices (prefix cache and LM head "
                "stay resident)")


class TreeWorkload(FlatWorkload):
    """Candidate-prefix tree: trie-packed tokens attend to the root cache, their
    ancestors and their own node; readout of each leaf over its siblings."""

    def __init__(self, cfg, dev, jev, torch):
        self.cfg, self.jev, self.torch = cfg, jev, torch
        tc = synth.tree_case(cfg, with_lm_head=False)
        self.tc = tc
        trie = jev.jev_tree_build(tc.seq_off, tc.toks, cfg.Lp)
        plan = jev.jev_tree_readout_plan(tc.seq_off, tc.toks, tc.score_from, trie["path_row"])
        self.trie, self.plan = trie, plan
        N = int(trie["tok_off"][-1])
        # exact key count of every tree token: root cache + ancestors + own node up to itself
        pos = np.concatenate([trie["pos0"][n] + np.arange(trie["tok_off"][n + 1] - trie["tok_off"][n])
                              for n in range(1, trie["n_nodes"])])
        keys = pos.astype(np.int64) + 1
        s = 2
        n_pairs = plan["pair_tok"].size
        self.work = dict(T=N, B=int(tc.seq_off.size - 1),
                         flops_attn=int(4 * cfg.Hq * cfg.d * keys.sum()),
                         flops_readout=2 * cfg.H * n_pairs,
                         bytes_attn=s * (2 * N * cfg.Hq * cfg.d + 2 * cfg.Lp * cfg.Hkv * cfg.d + 2 * N * cfg.Hkv * cfg.d) + 4 * N * cfg.Hq,
                         bytes_readout=s * (N * cfg.H + n_pairs * cfg.H) + 8 * n_pairs)
        self.T, self.B = N, self.work["B"]
        self.tdt = torch.bfloat16
        self.W = load_lm_head(cfg, dev, torch, self.tdt)
        self.base = dict(q=to_dev(tc.q, dev, torch), k_pre=to_dev(tc.k_root, dev, torch), v_pre=to_dev(tc.v_root, dev, torch),
                         k_suf=to_dev(tc.k, dev, torch), v_suf=to_dev(tc.v, dev, torch),
                         hidden=to_dev(tc.hidden, dev, torch), pair_tok=to_dev(plan["pair_tok"], dev, torch))
        self.parent = to_dev(trie["parent"], dev, torch)
        self.tok_off = to_dev(trie["tok_off"], dev, torch)
        self.pos0 = to_dev(trie["pos0"], dev, torch)
        self.co = to_dev(plan["cand_offsets"], dev, torch)
        self.prow = to_dev(plan["pair_row"], dev, torch)
        self.so = to_dev(tc.set_offsets, dev, torch)
        desc = jev.make_attn_desc(trie["n_nodes"] - 1, cfg.Lp, cfg.Hq, cfg.Hkv, cfg.d, N, jev.JEV_BF16, cfg.theta)
        self.ws = jev.new_workspace(jev.jev_tree_attn_workspace(desc, trie["n_nodes"]), dev)
        self.out = torch.empty_like(self.base["q"])
        self.lse = torch.empty((N, cfg.Hq), dtype=torch.float32, device=dev)
        self.lp = torch.empty(self.co.numel() - 1, dtype=torch.float32, device=dev)
        self.choice = torch.empty(self.so.numel() - 1, dtype=torch.int32, device=dev)
        self.e2e_inputs = ("q", "k_suf", "v_suf", "hidden")

    def attn(self, cp, s):
        self.jev.jev_tree_attn(cp.get("parent", self.parent), cp.get("tok_off", self.tok_off), cp.get("pos0", self.pos0),
                               cp["q"], cp["k_pre"], cp["v_pre"], cp["k_suf"], cp["v_suf"], out=self.out, lse=self.lse,
                               workspace=self.ws, rope_theta=self.cfg.theta, stream=s)

    def readout(self, cp, s):
        self.jev.jev_candidate_readout(cp["hidden"], self.W, cp.get("so", self.so), cp.get("pair_tok", self.base["pair_tok"]),
                                       cand_offsets=cp.get("co", self.co), pair_row=cp.get("prow", self.prow),
                                       logprob=self.lp, choice=self.choice, stream=s)

    def e2e_host(self):
        h = {k: self.base[k].cpu().pin_memory() for k in self.e2e_inputs}
        return h

    def host_prep(self, h):
        """The trie build and readout plan of the request run on the host every step."""
        tc, jev, t = self.tc, self.jev, self.torch
        trie = jev.jev_tree_build(tc.seq_off, tc.toks, self.cfg.Lp)
        plan = jev.jev_tree_readout_plan(tc.seq_off, tc.toks, tc.score_from, trie["path_row"])
        h = dict(h)
        for k, v in (("parent", trie["parent"]), ("tok_off", trie["tok_off"]), ("pos0", trie["pos0"]),
                     ("co", plan["cand_offsets"]), ("prow", plan["pair_row"]), ("pair_tok", plan["pair_tok"]),
                     ("so", tc.set_offsets)):
            h[k] = t.from_numpy(np.ascontiguousarray(v, dtype=np.int32))
        return h

    def describe_e2e(self):
        return ("per step: host trie build and readout plan written into a pinned staging buffer with the "
                "tree-token q/k/v and hidden rows; one H2D copy; both API calls; one D2H copy of log-probs and "
                "choices (root cache and LM head stay resident)")


def to_dev(a, dev, torch):
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev)


def load_lm_head(cfg, dev, torch, tdt):
    W = torch.empty((cfg.V, cfg.H), dtype=tdt, device=dev)
    for ch in range((cfg.V + synth.W_CHUNK_ROWS - 1) // synth.W_CHUNK_ROWS):
        blk = synth.lm_head_block(cfg.seed, cfg.V, cfg.H, ch, cfg.dtype, cfg.w_std)
        W[ch * synth.W_CHUNK_ROWS: ch * synth.W_CHUNK_ROWS + blk.shape[0]] = to_dev(blk, dev, torch)
    return W


def graph_us(torch, fn, stream, steps: int, warmup: int) -> float:
    """Average device time of fn() replayed from one CUDA graph, after warm-up."""
    stream.wait_stream(torch.cuda.current_stream())  # inputs were made on the current stream
    with torch.cuda.stream(stream):
        fn()
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn()
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            g.replay()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for _ in range(steps):
            g.replay()
        a1.record(stream)
    torch.cuda.synchronize()
    return 1e3 * a0.elapsed_time(a1) / steps


def diag_vocab_lse(dev, jev, torch, stream, W=None) -> dict:
    """Full-vocabulary LSE (normalised multi-token scoring): 256 hidden rows
    against the whole 7B-shaped LM head (152064 x 3584, N(0, 0.02)), graph-replayed."""
    cfg = synth.CONFIGS["wide_7b"]
    pk, _ = peaks()
    if W is None:
        W = load_lm_head(cfg, dev, torch, torch.bfloat16)
    rng = np.random.default_rng(8)
    R_l = 256
    hl = to_dev(synth.f32_to_bf16_bits(rng.standard_normal((R_l, cfg.H)).astype(np.float32)), dev, torch)
    lse_l = torch.empty(R_l, dtype=torch.float32, device=dev)
    ws_l = jev.new_workspace(jev.jev_vocab_lse_workspace(R_l, cfg.V), dev)
    us_l = graph_us(torch, lambda: jev.jev_vocab_lse(hl, W, lse=lse_l, workspace=ws_l,
                                                     stream=torch.cuda.current_stream()), stream, 20, 3)
    flags = jev.jev_check_device_status(ws_l)
    lflops = 2 * R_l * cfg.V * cfg.H
    lpeak = float(pk["bf16_tflops"])
    lsus = float(pk.get("bf16_tflops_sustained", lpeak))
    return {"workload": f"{R_l} rows x LM head {cfg.V} x {cfg.H}", "flops_per_call": lflops,
            "head_bytes": cfg.V * cfg.H * 2, "us": us_l, "TFLOPs": lflops / us_l / 1e6,
            "frac_of_burst_bf16": lflops / us_l / 1e6 / lpeak, "frac_of_sustained_bf16": lflops / us_l / 1e6 / lsus,
            "head_GBps": cfg.V * cfg.H * 2 / us_l / 1e3,
            "device_flags": flags,
            "note": "GEMM with an on-chip online LSE and the partial merge; no logits in HBM"}


def _tree_timer(dev, jev, torch, stream, tc) -> dict:
    """Graph-replayed time of one jev_tree_attn call over a synthetic trie, with its exact work."""
    cfg = tc.cfg
    trie = jev.jev_tree_build(tc.seq_off, tc.toks, cfg.Lp)
    parent, tok_off, pos0 = (to_dev(trie[k], dev, torch) for k in ("parent", "tok_off", "pos0"))
    q, kr, vr, k, v = (to_dev(x, dev, torch) for x in (tc.q, tc.k_root, tc.v_root, tc.k, tc.v))
    N = int(trie["tok_off"][-1])
    out = torch.empty_like(q)
    lse = torch.empty((N, cfg.Hq), dtype=torch.float32, device=dev)
    desc = jev.make_attn_desc(trie["n_nodes"] - 1, cfg.Lp, cfg.Hq, cfg.Hkv, cfg.d, N, jev.JEV_BF16, cfg.theta)
    ws = jev.new_workspace(jev.jev_tree_attn_workspace(desc, trie["n_nodes"]), dev)
    us = graph_us(torch, lambda: jev.jev_tree_attn(parent, tok_off, pos0, q, kr, vr, k, v, out=out, lse=lse,
                                                   workspace=ws, rope_theta=cfg.theta,
                                                   stream=torch.cuda.current_stream()), stream, 50, 5)
    pos = np.concatenate([trie["pos0"][n] + np.arange(trie["tok_off"][n + 1] - trie["tok_off"][n])
                          for n in range(1, trie["n_nodes"])])
    flops = int(4 * cfg.Hq * cfg.d * (pos.astype(np.int64) + 1).sum())
    logical = int(tc.seq_off[-1])
    return {"us": us, "unique_tokens": N, "logical_tokens": logical, "merged_frac": 1 - N / logical,
            "nodes": int(trie["n_nodes"]), "flops": flops, "TFLOPs": flops / us / 1e6,
            "device_flags": jev.jev_check_device_status(ws)}


def diag_tree_schedule(dev, jev, torch, stream) -> dict:
    """Tree schedule study at the 7B shape (root / prefix 2048 tokens, Hq 28, Hkv 4, d 128), after
    FastJEV §4.5 and §A.3: 64 candidates whose content is 75% shared, run as 64 flat branches
    (no merging) and as a two-level trie (16 questions of 24 tokens, 4 options of 8 tokens each);
    then a flat trie (64 disjoint 14-token candidates) with the same 896 unique tokens as the
    two-level trie.  Plus the multi-image variant (Ochevid, "One question, multiple images"):
    8 images of 400 tokens plus a 16-token question each, 3 one-token options, an empty root."""
    import dataclasses
    B, BF = synth.BF16, synth.CONFIGS["qwen25vl_7b"]
    res = {}
    # 64 flat branches of 32 tokens: 2048 suffix tokens, nothing merged
    fc = synth.flat_case(dataclasses.replace(BF, B=64), with_lm_head=False, lengths=np.full(64, 32, np.int32))
    a = [to_dev(x, dev, torch) for x in (fc.q, fc.k_pre, fc.v_pre, fc.k_suf, fc.v_suf)]
    cu = torch.from_numpy(fc.cu_seqlens).to(dev)
    desc = jev.make_attn_desc(64, BF.Lp, BF.Hq, BF.Hkv, BF.d, fc.T, jev.JEV_BF16, BF.theta)
    ws = jev.new_workspace(jev.jev_prefix_suffix_attn_workspace(desc), dev)
    o = torch.empty_like(a[0])
    lse = torch.empty((fc.T, BF.Hq), dtype=torch.float32, device=dev)
    us = graph_us(torch, lambda: jev.jev_prefix_suffix_attn(*a, cu, out=o, lse=lse, workspace=ws, rope_theta=BF.theta,
                                                            stream=torch.cuda.current_stream()), stream, 50, 5)
    fl = flat_work(fc)["flops_attn"]
    res["branches_64x32"] = {"us": us, "unique_tokens": fc.T, "logical_tokens": fc.T, "merged_frac": 0.0,
                             "flops": fl, "TFLOPs": fl / us / 1e6}
    two = synth.TreeConfig("two_level", B, BF.Lp, 16, 24, 4, 4, 8, 8, BF.Hq, BF.Hkv, BF.d, BF.H, BF.V, seed=31)
    res["trie_two_level_16x24_4x8"] = _tree_timer(dev, jev, torch, stream, synth.tree_case(two, with_lm_head=False))
    flat = synth.TreeConfig("flat_trie", B, BF.Lp, 64, 13, 1, 1, 1, 1, BF.Hq, BF.Hkv, BF.d, BF.H, BF.V, seed=32)
    res["trie_flat_64x14"] = _tree_timer(dev, jev, torch, stream, synth.tree_case(flat, with_lm_head=False))
    res["speedup_trie_vs_branches"] = res["branches_64x32"]["us"] / res["trie_two_level_16x24_4x8"]["us"]
    res["two_level_over_flat_trie_time"] = res["trie_two_level_16x24_4x8"]["us"] / res["trie_flat_64x14"]["us"]
    mi = synth.TreeConfig("multi_image", B, 0, 8, 416, 3, 3, 1, 1, BF.Hq, BF.Hkv, BF.d, BF.H, BF.V, seed=33)
    r = _tree_timer(dev, jev, torch, stream, synth.tree_case(mi, with_lm_head=False))
    r["images_per_s"] = 8 / (r["us"] / 1e6)
    res["multi_image_8x416"] = r
    return res


def diag_decode(dev, jev, torch, stream, names=("qwen25vl_7b", "wide_7b")) -> dict:
    """One generation step after the decision (jev_suffix_cache_attn): every
    branch of the workload appends one token over the shared prefix and its
    cached suffix (U[lo, hi] tokens, as drawn for the workload; cache rows
    packed with 8 spare rows per branch).  Graph-replayed; per-kernel times
    from a second replay with event nodes.  Attention FLOPs count the keys
    each new token sees: 4 * Hq * d * sum_b (Lp + cached_b + 1)."""
    pk, src = peaks()
    res = {}
    for name in names:
        cfg = synth.CONFIGS[name]
        Ls = synth.suffix_lengths(cfg)
        B = cfg.B
        rng = np.random.default_rng(9)
        mk = lambda *sh: to_dev(synth.f32_to_bf16_bits(rng.standard_normal(sh).astype(np.float32)), dev, torch)
        co = np.concatenate([[0], np.cumsum(Ls + 8)]).astype(np.int32)
        kc, vc = mk(int(co[-1]), cfg.Hkv, cfg.d), mk(int(co[-1]), cfg.Hkv, cfg.d)
        kp, vp = mk(cfg.Lp, cfg.Hkv, cfg.d), mk(cfg.Lp, cfg.Hkv, cfg.d)
        q, kn, vn = mk(B, cfg.Hq, cfg.d), mk(B, cfg.Hkv, cfg.d), mk(B, cfg.Hkv, cfg.d)
        cod, cld = torch.from_numpy(co).to(dev), torch.from_numpy(Ls).to(dev)
        cu = torch.arange(B + 1, dtype=torch.int32, device=dev)
        desc = jev.make_attn_desc(B, cfg.Lp, cfg.Hq, cfg.Hkv, cfg.d, B, jev.JEV_BF16, cfg.theta)
        ws = jev.new_workspace(jev.jev_suffix_cache_attn_workspace(desc), dev)
        out = torch.empty_like(q)
        lse = torch.empty((B, cfg.Hq), dtype=torch.float32, device=dev)

        def step():
            jev.jev_suffix_cache_attn(q, kn, vn, kp, vp, kc, vc, cod, cld, cu, out=out, lse=lse, workspace=ws,
                                      rope_theta=cfg.theta, stream=torch.cuda.current_stream())
        us = graph_us(torch, step, stream, 200, 10)
        jev.jev_profile_read()
        jev.jev_profile_enable(True)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            step()
        jev.jev_profile_enable(False)
        with torch.cuda.stream(stream):
            for _ in range(3):
                g.replay()
        torch.cuda.synchronize()
        prof = {k: 1e3 * v[1] / max(v[0], 1) for k, v in jev.jev_profile_read().items()}
        del g
        flops = 4 * cfg.Hq * cfg.d * int((cfg.Lp + Ls.astype(np.int64) + 1).sum())
        res[name] = {"branches": B, "cached_tokens": int(Ls.sum()), "us_per_step": us,
                     "new_tokens_per_s": B / (us / 1e6), "kernels_us": prof, "flops_per_step": flops,
                     "TFLOPs": flops / us / 1e6, "device_flags": jev.jev_check_device_status(ws)}
    return res


def diag_attn(dev, jev, torch, stream, wl_name: str) -> dict:
    """The workload's attention call alone (no LM head on the device, one set
    of inputs): a small case for ncu captures of the attention kernels.
    Runs 3 warm-up calls, then 3 calls between CUDA events."""
    cfg = synth.CONFIGS[wl_name]
    if isinstance(cfg, synth.TreeConfig):
        tc = synth.tree_case(cfg, with_lm_head=False)
        trie = jev.jev_tree_build(tc.seq_off, tc.toks, cfg.Lp)
        parent, tok_off, pos0 = (to_dev(trie[k], dev, torch) for k in ("parent", "tok_off", "pos0"))
        q, kr, vr, k, v = (to_dev(x, dev, torch) for x in (tc.q, tc.k_root, tc.v_root, tc.k, tc.v))
        out = torch.empty_like(q)

        def call():
            jev.jev_tree_attn(parent, tok_off, pos0, q, kr, vr, k, v, out=out, rope_theta=cfg.theta, stream=stream)
    else:
        c = synth.flat_case(cfg, with_lm_head=False)
        a = [to_dev(x, dev, torch) for x in (c.q, c.k_pre, c.v_pre, c.k_suf, c.v_suf)]
        cu = torch.from_numpy(c.cu_seqlens).to(dev)
        out = torch.empty_like(a[0])
        desc = jev.make_attn_desc(cfg.B, cfg.Lp, cfg.Hq, cfg.Hkv, cfg.d, c.T,
                                  jev.JEV_BF16 if cfg.dtype == synth.BF16 else jev.JEV_F32, cfg.theta)
        ws = jev.new_workspace(jev.jev_prefix_suffix_attn_workspace(desc), dev)

        def call():
            jev.jev_prefix_suffix_attn(*a, cu, out=out, workspace=ws, rope_theta=cfg.theta, stream=stream)
    torch.cuda.synchronize()
    for _ in range(3):
        call()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(3):
        call()
    e1.record(stream)
    torch.cuda.synchronize()
    return {"workload": wl_name, "us_per_call": 1e3 * e0.elapsed_time(e1) / 3,
            "note": "direct launches, not graph-replayed; for profiling captures, not a bench number"}


def diag_readout(dev, jev, torch, stream, W=None) -> dict:
    """The readout over 4096 option sets of 9 one-token options at the 7B
    shape (H = 3584, V = 152064): the option rows of the LM head gathered from
    HBM, one warp per set, scores and set softmax fused."""
    pk, _ = peaks()
    hbm = float(pk["hbm_gbs"])
    cfg = synth.CONFIGS["wide_7b"]
    if W is None:
        W = load_lm_head(cfg, dev, torch, torch.bfloat16)
    n_sets, opts = 4096, 9
    rng = np.random.default_rng(7)
    hidden = to_dev(synth.f32_to_bf16_bits(rng.standard_normal((n_sets, cfg.H)).astype(np.float32)), dev, torch)
    base = rng.integers(0, cfg.V, n_sets)
    toks = ((base[:, None] + 16411 * np.arange(opts)[None, :]) % cfg.V).astype(np.int32).reshape(-1)
    so = torch.arange(0, n_sets * opts + 1, opts, dtype=torch.int32, device=dev)
    pt = torch.from_numpy(toks).to(dev)
    lp = torch.empty(toks.size, dtype=torch.float32, device=dev)
    ch = torch.empty(n_sets, dtype=torch.int32, device=dev)
    us = graph_us(torch, lambda: jev.jev_candidate_readout(hidden, W, so, pt, logprob=lp, choice=ch,
                                                           stream=torch.cuda.current_stream()), stream, 200, 10)
    nbytes = (toks.size + n_sets) * cfg.H * 2 + toks.size * 8 + n_sets * 4
    return {"sets": n_sets, "options": opts, "H": cfg.H, "bytes_per_call": nbytes, "us": us,
            "GBps": nbytes / us / 1e3, "frac_of_hbm": nbytes / us / 1e3 / hbm,
            "note": "option rows of the LM head gathered from HBM; one kernel (scores and set softmax fused)"}


def diagnostics(dev, jev, torch) -> dict:
    """Streaming efficiency of the HBM-bound kernels at sizes where it can be
    measured (the configs move kilobytes to a few megabytes per launch, below
    launch latency): the readout over 4096 option sets of 9 one-token options
    at the 7B shape (H = 3584, V = 152064), and the RoPE pack at the wide
    shape with 1024 branches.  Inputs are synthetic and seeded."""
    import dataclasses
    pk, src = peaks()
    hbm = float(pk["hbm_gbs"])
    out = {"peak_hbm_GBps": hbm, "peak_source": src}
    stream = torch.cuda.Stream(device=dev)
    # ---- readout
    cfg = synth.CONFIGS["wide_7b"]
    W = load_lm_head(cfg, dev, torch, torch.bfloat16)
    rng = np.random.default_rng(7)
    out["readout"] = diag_readout(dev, jev, torch, stream, W)
    out["vocab_lse"] = diag_vocab_lse(dev, jev, torch, stream, W)
    del W
    torch.cuda.empty_cache()
    out["tree_schedule"] = diag_tree_schedule(dev, jev, torch, stream)
    torch.cuda.empty_cache()
    out["decode_step"] = diag_decode(dev, jev, torch, stream)
    torch.cuda.empty_cache()
    # ---- RoPE pack (and the attention call around it) at the wide shape with 1024 branches
    cw = dataclasses.replace(synth.CONFIGS["wide_7b"], B=1024)
    c = synth.flat_case(cw, with_lm_head=False)
    args_ = [to_dev(x, dev, torch) for x in (c.q, c.k_pre, c.v_pre, c.k_suf, c.v_suf)]
    cu = torch.from_numpy(c.cu_seqlens).to(dev)
    desc = jev.make_attn_desc(cw.B, cw.Lp, cw.Hq, cw.Hkv, cw.d, c.T, jev.JEV_BF16, cw.theta)
    ws = jev.new_workspace(jev.jev_prefix_suffix_attn_workspace(desc), dev)
    o = torch.empty_like(args_[0])
    lse = torch.empty((c.T, cw.Hq), dtype=torch.float32, device=dev)

    def attn():
        jev.jev_prefix_suffix_attn(*args_, cu, out=o, lse=lse, workspace=ws, rope_theta=cw.theta,
                                   stream=torch.cuda.current_stream())
    graph_us(torch, attn, stream, 3, 2)  # warm-up, no profiling
    # per-kernel times: one graph with event nodes around each kernel, replayed
    jev.jev_profile_read()
    jev.jev_profile_enable(True)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        attn()
    jev.jev_profile_enable(False)
    with torch.cuda.stream(stream):
        for _ in range(3):
            g.replay()
    torch.cuda.synchronize()
    prof = jev.jev_profile_read()
    del g
    # the pack reads q and k and writes their rotated copies (bf16), plus 16 bytes of token info
    rbytes = 2 * 2 * c.T * (cw.Hq + cw.Hkv) * cw.d + 16 * c.T
    n_l, t_ms = prof.get("rope_pack", (1, float("nan")))
    rus = 1e3 * t_ms / max(n_l, 1)
    out["rope_pack"] = {"workload": f"wide shape, B=1024 ({c.T} suffix tokens)", "bytes_per_call": rbytes,
                        "us": rus, "GBps": rbytes / rus / 1e3, "frac_of_hbm": rbytes / rus / 1e3 / hbm,
                        "note": "per-kernel event time (includes launch latency)"}
    out["attn_call_us"] = {k: 1e3 * v[1] / max(v[0], 1) for k, v in prof.items()}
    del args_, o, lse, ws
    torch.cuda.empty_cache()
    # ---- sink-block parallel encoding (flat kernels, sequential positions): 32 blocks of 1024 tokens over a
    # 64-token sink
    S, nb, bl, Hq, Hkv, d = 64, 32, 1024, 28, 4, 128
    cu_sb = np.arange(0, nb * bl + 1, bl, dtype=np.int32)
    Tsb = nb * bl
    mk = lambda *sh: to_dev(synth.f32_to_bf16_bits(rng.standard_normal(sh).astype(np.float32)), dev, torch)
    sq, sk, sv, ssk, ssv = mk(Tsb, Hq, d), mk(Tsb, Hkv, d), mk(Tsb, Hkv, d), mk(S, Hkv, d), mk(S, Hkv, d)
    cu_d = torch.from_numpy(cu_sb).to(dev)
    sdesc = jev.make_attn_desc(nb, S, Hq, Hkv, d, Tsb, jev.JEV_BF16, pos_mode=1)
    sws = jev.new_workspace(jev.jev_prefix_suffix_attn_workspace(sdesc), dev)
    so_, sl_ = torch.empty_like(sq), torch.empty((Tsb, Hq), dtype=torch.float32, device=dev)

    def sink_block():
        jev.jev_sink_block_attn(sq, ssk, ssv, sk, sv, cu_d, out=so_, lse=sl_, workspace=sws,
                                stream=torch.cuda.current_stream())
    graph_us(torch, sink_block, stream, 3, 2)
    jev.jev_profile_read()
    jev.jev_profile_enable(True)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        sink_block()
    jev.jev_profile_enable(False)
    with torch.cuda.stream(stream):
        for _ in range(3):
            g.replay()
    torch.cuda.synchronize()
    sprof = jev.jev_profile_read()
    del g
    sflops = 4 * Hq * d * nb * (bl * S + bl * (bl + 1) // 2)
    speak = float(pk["bf16_tflops"])
    s_us = {k: 1e3 * v[1] / max(v[0], 1) for k, v in sprof.items()}
    if "attn_tc" in s_us:
        out["sink_block"] = {"workload": f"{nb} blocks of {bl} tokens over a {S}-token sink, Hq={Hq}, Hkv={Hkv}, "
                                         f"d={d}", "flops_per_call": sflops, "kernels_us": s_us,
                             "TFLOPs": sflops / s_us["attn_tc"] / 1e6,
                             "frac_of_burst_bf16": sflops / s_us["attn_tc"] / 1e6 / speak,
                             "tokens_per_s": Tsb / (sum(s_us.values()) / 1e6)}
    # the tensor-core kernel at the wide size: many waves of whole tiles
    if "attn_tc" in prof:
        flops = flat_work(c)["flops_attn"]
        aus = out["attn_call_us"]["attn_tc"]
        peak = float(pk["bf16_tflops"])
        out["attn_tc"] = {"workload": out["rope_pack"]["workload"], "flops_per_call": flops, "us": aus,
                          "TFLOPs": flops / aus / 1e6, "frac_of_burst_bf16": flops / aus / 1e6 / peak}
    return out


def max_over_ranks(ms: float, dist, device, world: int) -> float:
    """This rank's device-timed milliseconds -> the slowest rank's, on every rank."""
    if world > 1:
        import torch
        t = torch.tensor([ms], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    return ms


def job_rate(world: int, units_per_rank_step: float, steps: int, ms: float) -> float:
    """Whole-job throughput: the units every rank processed over the slowest rank's time."""
    return world * units_per_rank_step * steps / (ms / 1e3)


class Measured:
    """One workload on this GPU: graphs over rotating input copies, the
    device-timed loop, and a second pass with per-kernel event nodes."""

    def __init__(self, wl_name, steps, warmup, world, dev, jev, torch, dist, clocks=None):
        self.cfg = cfg = synth.CONFIGS[wl_name]
        self.name, self.steps, self.warmup, self.world = wl_name, steps, warmup, world
        self.jev, self.torch, self.dist, self.dev = jev, torch, dist, dev
        self.wl = wl = (TreeWorkload if isinstance(cfg, synth.TreeConfig) else FlatWorkload)(cfg, dev, jev, torch)
        # ---- device copies of the per-step inputs, enough to exceed twice the L2
        self.per_copy = sum(t.numel() * t.element_size() for t in wl.base.values())
        self.ncopies = max(2, math.ceil(2 * L2_BYTES / self.per_copy))
        self.copies = []
        for i in range(self.ncopies):
            cp = {k: v.clone() for k, v in wl.base.items()}
            # each copy reads different option rows of the LM head
            cp["pair_tok"] = ((wl.base["pair_tok"].long() + 7919 * i) % cfg.V).to(torch.int32)
            self.copies.append(cp)
        self.stream = torch.cuda.Stream(device=dev)
        self.side = torch.cuda.Stream(device=dev)
        with torch.cuda.stream(self.stream):
            for i in range(3):
                self.step(self.copies[i % self.ncopies], self.stream)
        self.stream.synchronize()
        self.ngraph = max(1, min(self.ncopies, steps))
        graphs, self.launches_per_step = self.capture(False)
        if clocks:
            clocks.start()
        self.ms = self.timed_loop(graphs)
        self.clk = clocks.stop() if clocks else None
        self.ms = self.max_over_ranks(self.ms)
        assert jev.jev_check_device_status(wl.ws, self.stream) == 0, "device status flags set during the bench"
        # per-step spread: up to 500 more steps, each between its own pair of events
        n = min(steps, 500)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        with torch.cuda.stream(self.stream):
            for i, (e0, e1) in enumerate(evs):
                e0.record(self.stream)
                graphs[i % self.ngraph].replay()
                e1.record(self.stream)
        torch.cuda.synchronize()
        per = sorted(1e3 * e0.elapsed_time(e1) for e0, e1 in evs)
        self.pct = {"p10": per[n // 10], "p50": per[n // 2], "p90": per[(9 * n) // 10], "steps": n,
                    "note": "each step between its own pair of events, which adds a few microseconds"}
        del graphs
        # ---- per-kernel durations: the same K steps replayed from graphs whose
        # kernels are bracketed by CUDA event nodes on the launching stream; each
        # graph's events hold its last replay, one sample per input copy
        jev.jev_profile_read()
        pgraphs, _ = self.capture(True)
        self.prof_ms = self.timed_loop(pgraphs)
        self.prof = jev.jev_profile_read()
        del pgraphs

    def step(self, cp, s):
        # the readout's inputs (final hidden rows, option ids) do not depend on
        # this attention layer, so it runs on a second stream, forked and
        # joined inside the step.  It is enqueued after the attention kernels
        # so that their persistent CTAs take the SMs first and the readout's
        # blocks fill SMs as the attention's tail frees them (measured about
        # 1% faster per step than launching the readout first).
        self.side.wait_stream(s)
        self.wl.attn(cp, s)
        self.wl.readout(cp, self.side)
        s.wait_stream(self.side)

    def capture(self, profiled: bool):
        torch, jev = self.torch, self.jev
        jev.jev_profile_enable(profiled)
        n0 = jev.jev_launch_count()
        gs = []
        for cp in self.copies[:self.ngraph]:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=self.stream):
                self.step(cp, torch.cuda.current_stream())
            gs.append(g)
        jev.jev_profile_enable(False)
        return gs, (jev.jev_launch_count() - n0) // self.ngraph

    def timed_loop(self, gs):
        torch = self.torch
        with torch.cuda.stream(self.stream):
            for i in range(self.warmup):
                gs[i % self.ngraph].replay()
        self.stream.synchronize()
        if self.world > 1:
            self.dist.barrier()
        torch.cuda.synchronize()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(self.stream):
            a0.record(self.stream)
            for i in range(self.steps):
                gs[i % self.ngraph].replay()
            a1.record(self.stream)
        torch.cuda.synchronize()
        if self.world > 1:
            self.dist.barrier()
        return a0.elapsed_time(a1)

    def max_over_ranks(self, ms):
        return max_over_ranks(ms, self.dist, self.dev, self.world)

    def value(self):
        return job_rate(self.world, self.wl.T, self.steps, self.ms)

    def summary(self):
        """Per-kernel times and the roofline of the attention kernel."""
        pk, src = peaks()
        prof, work = self.prof, self.wl.work
        attn_name = "attn_tc" if "attn_tc" in prof else "attn_simt"
        dom = max(prof.items(), key=lambda kv: kv[1][1])[0] if prof else attn_name
        n_l, t_ms = prof.get(attn_name, (1, float("nan")))
        achieved = work["flops_attn"] / (t_ms / 1e3 / max(n_l, 1)) / 1e12
        # the kernel is event-timed over launches of tens to hundreds of
        # microseconds at full clock: the burst GEMM figure is its peak
        peak = float(pk["bf16_tflops"])
        sustained = float(pk.get("bf16_tflops_sustained", peak))
        tot_prof = sum(x[1] for x in prof.values()) or 1.0
        per_kernel = {k: {"launches": v[0], "avg_us": 1e3 * v[1] / max(v[0], 1), "share": v[1] / tot_prof}
                      for k, v in prof.items()}
        step_s = self.ms / 1e3 / self.steps
        ideal = max((work["flops_attn"] + work["flops_readout"]) / (float(pk["bf16_tflops"]) * 1e12),
                    (work["bytes_attn"] + work["bytes_readout"]) / (float(pk["hbm_gbs"]) * 1e9))
        roof = {"bound": "tensor", "kernel": attn_name, "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": traffic_of(attn_name, self.name, KERNEL_SRC[attn_name]),
                "peak_source": f"bf16_tflops (burst), {src}",
                "frac_of_sustained_peak": achieved / sustained,
                "algorithmic_flops_per_launch": work["flops_attn"], "dominant_kernel_by_time": dom}
        step_roof = {"ideal_us": ideal * 1e6, "measured_us": step_s * 1e6, "frac": ideal / step_s,
                     "definition": "max(F / bf16 burst peak, U / HBM peak) over the whole step"}
        return roof, step_roof, per_kernel

    def free(self):
        del self.copies, self.wl
        self.torch.cuda.empty_cache()


def jev_arm(args, wl_name):
    import torch
    import torch.distributed as dist
    import attention_cascade_b200 as jev

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)
    m = Measured(wl_name, args.steps, args.warmup, world, dev, jev, torch, dist, ClockSampler(local))
    wl, cfg, ms, T = m.wl, m.cfg, m.ms, m.wl.T

    # ---- end to end through the public API: pinned host inputs in, results out, every step.
    # Every per-step input sits in one pinned staging buffer (256-byte aligned
    # views) and goes to the device in one copy; both results come back in one.
    # Two staging slots: step i's upload runs on a copy stream into slot i % 2
    # while step i - 1 computes from the other slot (the copy engine and the
    # SMs overlap, as a serving loop would run them).
    hq = wl.e2e_host()
    first = wl.host_prep(hq)
    offs, total = {}, 0
    for k, v in first.items():
        off = (total + 255) // 256 * 256
        offs[k] = (off, v.dtype, tuple(v.shape))
        total = off + v.numel() * v.element_size()

    def views(buf):
        out = {}
        for k, (off, dt, shp) in offs.items():
            n = math.prod(shp) * torch.empty((), dtype=dt).element_size()
            out[k] = buf[off:off + n].view(dt).view(shp)
        return out

    n_slots = 2
    h_packs = [torch.empty(total, dtype=torch.uint8).pin_memory() for _ in range(n_slots)]
    d_packs = [torch.empty(total, dtype=torch.uint8, device=dev) for _ in range(n_slots)]
    h_ins, d_ins = [views(b) for b in h_packs], [views(b) for b in d_packs]
    for hi in h_ins:
        for k, v in first.items():
            hi[k].copy_(v)
    n_lp, n_ch = wl.lp.numel(), wl.choice.numel()
    lp_bytes = (n_lp * 4 + 255) // 256 * 256
    d_out = torch.empty(lp_bytes + n_ch * 4, dtype=torch.uint8, device=dev)
    wl.lp, wl.choice = d_out[:n_lp * 4].view(torch.float32), d_out[lp_bytes:].view(torch.int32)
    h_out = torch.empty(d_out.numel(), dtype=torch.uint8).pin_memory()
    cp_static = {k: v for k, v in wl.base.items() if k in ("k_pre", "v_pre")}
    copy_stream = torch.cuda.Stream(device=dev)
    uploaded = [torch.cuda.Event() for _ in range(n_slots)]  # the slot's inputs are on the device
    consumed = [torch.cuda.Event() for _ in range(n_slots)]  # the slot's step has finished with them
    step_no = [0]

    def e2e_step(s):
        slot = step_no[0] % n_slots
        step_no[0] += 1
        h = wl.host_prep(hq)
        if h is not hq:  # host-built arrays of this step (the tree's trie and readout plan)
            uploaded[slot].synchronize()  # the slot's previous upload has left the host buffer
            for k, v in h.items():
                if k not in hq:
                    h_ins[slot][k].copy_(v)
        copy_stream.wait_event(consumed[slot])
        with torch.cuda.stream(copy_stream):
            d_packs[slot].copy_(h_packs[slot], non_blocking=True)
        uploaded[slot].record(copy_stream)
        s.wait_event(uploaded[slot])
        cp = dict(cp_static)
        cp.update(d_ins[slot])
        m.step(cp, s)
        consumed[slot].record(s)
        h_out.copy_(d_out, non_blocking=True)

    stream = m.stream
    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            e2e_step(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        f0.record(stream)
        copy_stream.wait_stream(stream)  # no upload of the timed steps starts before f0
        for _ in range(args.steps):
            e2e_step(stream)
        f1.record(stream)
    torch.cuda.synchronize()
    # the pipelined steps computed what a step computes alone: the last step's
    # results, read back, against one more step run by itself from a slot
    # (every kernel on this path is deterministic)
    last = h_out.clone()
    with torch.cuda.stream(stream):
        cp = dict(cp_static)
        cp.update(d_ins[0])
        m.step(cp, stream)
        h_out.copy_(d_out, non_blocking=True)
    torch.cuda.synchronize()
    if not torch.equal(last, h_out):
        raise SystemExit("bench.py: end-to-end results differ from a step run alone")
    e2e_ms = m.max_over_ranks(f0.elapsed_time(f1))
    h2d = h_packs[0].numel()
    d2h = h_out.numel()

    roof, step_roof, per_kernel = m.summary()
    line = {
        "metric": METRIC, "value": m.value(), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "step_us_spread": m.pct,
        "vs_baseline": None, "dtype": "bf16" if cfg.dtype == synth.BF16 else "f32", "data": "synthetic",
        "config": bench_config(wl_name, world, T, wl.B),
        "method": {"l2": f"inputs rotate over {m.ngraph} device copies ({m.ngraph * m.per_copy / 2**20:.0f} MiB "
                         "> 2x L2)",
                   "timing": "CUDA graph replay per step, CUDA events on the launching stream; per-kernel times "
                             "from a second replay of the K steps with event nodes around each kernel",
                   "streams": "readout on a second stream, forked before and enqueued after the attention kernels, joined inside each step"},
        "branches_per_s": job_rate(world, wl.B, args.steps, ms),
        "clocks": m.clk,
        "e2e": {"value": job_rate(world, T, args.steps, e2e_ms), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "note": wl.describe_e2e() + "; two staging slots: each step's H2D copy runs on a copy stream "
                                            "and overlaps the previous step's kernels"},
        "gpu_launches": m.launches_per_step * args.steps,
        "roofline": roof,
        "step_roofline": step_roof,
        "kernels": per_kernel,
        "profiled_pass_ms_per_step": m.prof_ms / args.steps,
    }
    m.free()
    del m

    # ---- the other synthetic configs, same method, fewer steps (one GPU only)
    if world == 1 and args.per_config:
        per = {}
        for name in sorted(synth.CONFIGS):
            if name == wl_name:
                continue
            steps = max(50, min(args.steps, args.per_config_steps))
            mc = Measured(name, steps, args.warmup, 1, dev, jev, torch, dist)
            r, sr, pk_ = mc.summary()
            per[name] = {"workload": synth.WORKLOAD_TEXT[name], "value": mc.value(), "unit": "tokens/s",
                         "ms_per_step": mc.ms / steps, "steps": steps,
                         "branches_per_s": mc.wl.B * steps / (mc.ms / 1e3),
                         "dtype": "bf16" if mc.cfg.dtype == synth.BF16 else "f32",
                         "roofline": {k: r[k] for k in ("bound", "kernel", "achieved", "peak", "unit", "frac",
                                                        "traffic", "peak_source", "frac_of_sustained_peak")},
                         "step_roofline_frac": sr["frac"],
                         "kernels": {k: round(v["avg_us"], 2) for k, v in pk_.items()}}
            mc.free()
            del mc
            if os.environ.get("JEV_SKIP_CPU_BASELINE") != "1":
                per[name]["cpu_baseline"] = cpu_baseline(synth.CONFIGS[name],
                                                         float(os.environ.get("JEV_CPU_BASELINE_CONFIG_S", "5")))
        line["per_config"] = per
    if world == 1 and args.diagnostics:
        line["diagnostics"] = diagnostics(dev, jev, torch)

    if rank == 0 and world == 1 and os.environ.get("JEV_SKIP_CPU_BASELINE") != "1":
        line["cpu_baseline"] = cpu_baseline(cfg, float(os.environ.get("JEV_CPU_BASELINE_S", "12")))
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    # the default is the largest single-GPU workload
    ap.add_argument("--workload", default="wide_7b", choices=sorted(synth.CONFIGS))
    ap.add_argument("--impl", default="jev", choices=["jev", "reference"])
    ap.add_argument("--no-per-config", dest="per_config", action="store_false",
                    help="skip the other synthetic configs (reported under per_config on one GPU)")
    ap.add_argument("--per-config-steps", type=int, default=2000)
    ap.add_argument("--no-diagnostics", dest="diagnostics", action="store_false",
                    help="skip the streaming diagnostics at larger sizes (one GPU)")
    ap.add_argument("--diag", choices=["vocab_lse", "tree_schedule", "attn", "decode", "readout"], default=None,
                    help="run only this diagnostic on cuda:0 and print its JSON (a small case for profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("bench.py: at least 3 warm-up steps")
    if args.diag:
        import torch
        import attention_cascade_b200 as jev
        torch.cuda.set_device(0)
        stream = torch.cuda.Stream(device="cuda:0")
        if args.diag == "attn":
            res = diag_attn("cuda:0", jev, torch, stream, args.workload)
        else:
            fn = {"vocab_lse": diag_vocab_lse, "tree_schedule": diag_tree_schedule, "decode": diag_decode,
                  "readout": diag_readout}[args.diag]
            res = fn("cuda:0", jev, torch, stream)
        print(json.dumps({"diagnostic": args.diag, **res}))
    elif args.impl == "reference":
        reference_arm(args, args.workload)
    else:
        jev_arm(args, args.workload)


if __name__ == "__main__":
    main()
