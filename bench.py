"""Benchmark: block-sparse masked attention forward on B200.

One step is the whole hot path on one batch of synthetic input:
  1. the block-mask builder kernel (mask evaluation, tile classification,
     index compaction);
  2. the attention kernel over the tiles the mask keeps (score_mod and, on
     partial tiles only, mask_mod; online softmax; out and lse).

metric: TFLOP/s counting only the FLOPs of tiles that are not skipped,
4 * 128 * 128 * D per kept (FULL or PARTIAL) 128x128 tile per (b, hq).

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                       [--workload INDEX] [--no-cpu-baseline] [--backward-only] [--batch B]
For N > 1 run it under torch.distributed.run. Each rank then processes its
own batch of the same shape (weak scaling; the units are independent).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "flex_attention fwd TFLOP/s (unmasked tiles) and % of B200 BF16 tensor peak"
UNIT = "TFLOP/s"
DATASHEET_BF16_TFLOPS = 2250.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# the device sources the forward kernel is compiled from: a profile taken on
# other sources no longer describes it, and its DRAM traffic is not reported
ATTN_SOURCES = ["attn_fwd.cuh", "ptx.cuh", "mask_dnf.cuh"]


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", type=int, default=5)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-side-kernels", action="store_true",
                    help="skip the side measurements (builder, transpose, split-KV, varlen) after the step")
    ap.add_argument("--backward-only", action="store_true",
                    help="run only the backward (prep, dk/dv and dq kernels) --steps times after one forward, "
                         "and print its timing (for profiling the backward kernels)")
    ap.add_argument("--builder-only", action="store_true",
                    help="run only the block-mask builder --steps times at the workload's shape (--batch and "
                         "--heads override B and H) and print its timing (for profiling the builder)")
    ap.add_argument("--heads", type=int, default=0, help="override H for --builder-only")
    ap.add_argument("--batch", type=int, default=0,
                    help="override the workload's batch size (smaller cases for profiling only)")
    return ap.parse_args(argv)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            d = json.load(fh)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def attn_source_hash() -> str:
    h = hashlib.sha256()
    for f in ATTN_SOURCES:
        with open(os.path.join(ROOT, "block_sparse_masked_tile_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profile_figures(workload_name: str) -> dict:
    """Figures of the committed ncu summary of the attention kernel (DRAM bytes
    per launch, tensor and MUFU pipe shares of active cycles), if it was taken
    on the current kernel source (same hash); otherwise None for each."""
    keys = {"traffic": "dram_bytes_per_launch", "tensor_pipe_pct": "tensor_pipe_pct_active",
            "mufu_pipe_pct": "mufu_pipe_pct_active"}
    res = dict.fromkeys(keys)
    path = os.path.join(ROOT, "profiles", f"attn_fwd_{workload_name}.md")
    if not os.path.exists(path):
        return res
    text = open(path).read()
    m_hash = re.search(r"kernel_source_sha256_16:\s*([0-9a-f]+)", text)
    if not m_hash or m_hash.group(1) != attn_source_hash():
        return res
    for k, tag in keys.items():
        m = re.search(tag + r":\s*([0-9.eE+]+)", text)
        res[k] = float(m.group(1)) if m else None
    return res


def reduce_over_ranks(dist, device, times_ms, units):
    """Max over ranks of each time and sum over ranks of the work units.

    Every rank takes the same two all-reduces in the same order and gets the
    same result. ``dist`` is None for a single process."""
    t = torch.tensor([float(x) for x in times_ms], dtype=torch.float64, device=device)
    u = torch.tensor([float(units)], dtype=torch.float64, device=device)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        dist.all_reduce(u, op=dist.ReduceOp.SUM)
    return [float(x) for x in t], float(u[0])


class ClockSampler:
    """nvidia-smi clock / throttle sampling around the timed region.

    Samples arrive every 20 ms; each is stamped with the host's monotonic
    clock when it is read. ``mark_start`` / ``mark_end`` bracket the timed
    region, and ``summary`` keeps the samples read inside it (plus one
    interval after its end, the sample that covers its last stretch). A
    region shorter than the interval may hold none: then the summary uses
    every sample of the sampler's life and says so (``in_window`` false)."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    INTERVAL_MS = 20

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines: list[tuple[float, str]] = []
        self.t0 = self.t1 = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", str(self.INTERVAL_MS)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            deadline = time.monotonic() + 3.0
            while not self.lines and time.monotonic() < deadline:  # the sampler is running
                time.sleep(0.005)
        except FileNotFoundError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.monotonic(), line.strip()))

    def mark_start(self):
        self.t0 = time.monotonic()

    def mark_end(self):
        self.t1 = time.monotonic()
        time.sleep(2 * self.INTERVAL_MS / 1000)  # let the sample that covers the region's end arrive

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        in_window = [ln for t, ln in self.lines
                     if self.t0 is not None and self.t1 is not None and
                     self.t0 <= t <= self.t1 + self.INTERVAL_MS / 1000]
        chosen = in_window if in_window else [ln for _, ln in self.lines]
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in chosen:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        window_ms = None if self.t0 is None or self.t1 is None else round((self.t1 - self.t0) * 1e3, 1)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0, "in_window": False,
                    "window_ms": window_ms, "interval_ms": self.INTERVAL_MS}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm),
                "in_window": bool(in_window), "window_ms": window_ms, "interval_ms": self.INTERVAL_MS}


def _time_launches(fn, reps: int = 20) -> float:
    """Mean ms per call of fn: reps calls are captured in a CUDA graph (so the
    host's launch cost stays out), and the graph replay is timed with CUDA
    events on the replay stream."""
    for _ in range(3):
        fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(reps):
            fn()
    g.replay()
    torch.cuda.synchronize()
    s = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for _ in range(3):
        g.replay()
    e1.record(s)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / (3 * reps)
    del g
    return ms


BWD_PRODUCTS = 5  # dQ, dK, dV and the recomputed S and dP: 2*128*128*D FLOPs each per kept tile


def time_backward(bsmt, w, q, k, v, out, lse, bm, mods, dev, flops_fwd: int, reps: int = 5) -> dict:
    """The backward (prep + dk/dv + dq kernels) on the step's inputs, timed as
    CUDA-graph replays. Counted FLOPs: BWD_PRODUCTS products of 2*128*128*D per
    kept tile, i.e. 2.5x the forward count; the two kernels execute 7 products
    (S and dP are computed by both)."""
    g = torch.Generator(device="cpu").manual_seed(w.seed + 50)
    dout = torch.randn(out.shape, generator=g).to(torch.bfloat16).to(dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(bsmt.backward_workspace_bytes(w.B, w.Hq, w.M), dtype=torch.uint8, device=dev)
    bm.q_side()
    # ALiBi slopes on the device before capture (no host copies inside the graph)
    mods = [bsmt.ScoreMod(m.kind, m.value, None if m.slopes is None else m.slopes.to(dev)) for m in mods]

    def call():
        bsmt.flex_attention_backward(q, k, v, out, lse, dout, block_mask=bm, score_mod=mods, scale=w.scale,
                                     enable_gqa=w.enable_gqa, workspace=ws, dq=dq, dk=dk, dv=dv)

    ms = _time_launches(call, reps=reps)
    bsmt.check_device_status(dev)
    flops = flops_fwd * BWD_PRODUCTS // 2
    return {"ms": ms, "tflops": flops / (ms * 1e-3) / 1e12, "counted_gflop": flops / 1e9,
            "executed_tensor_tflops": flops * 7 / 5 / (ms * 1e-3) / 1e12,
            "note": "flex_attention_backward: lse/delta prep, dk/dv kernel (q-side lists), dq kernel (kv-side "
                    "lists); counted as 5 products per kept tile (2.5x forward)"}


def side_kernels(bsmt, mask, w, dev, hbm_peak: float) -> dict:
    """The HBM-bound kernels timed alone (outside the step): the block-mask
    builder at the step's shape and at B=8, H=32 (outputs larger than L2), and
    the q-side transpose. Algorithmic bytes are the outputs written: two count
    tensors and two index tensors."""
    import ctypes
    res = {}
    for label, B, H in (("mask_build", w.B, w.Hq), ("mask_build_b8_h32", 8, 32)):
        if w.mask == "doc_causal" and B != w.B:
            continue  # document ids are per batch row of the workload
        bm = bsmt.create_block_mask(mask, B, H, w.M, w.N, device=dev)
        ms = _time_launches(lambda: bsmt.create_block_mask(mask, B, H, w.M, w.N, device=dev, out=bm))
        Bm, Hm, QB, KB = bm.shape
        nbytes = 2 * 4 * Bm * Hm * QB + 2 * 4 * Bm * Hm * QB * KB
        gbs = nbytes / (ms * 1e-3) / 1e9
        res[label] = {"B": Bm, "H": Hm, "ms": ms, "bytes": nbytes, "achieved_gbs": gbs, "peak_gbs": hbm_peak,
                      "frac": gbs / hbm_peak, "note": "outputs larger than L2" if nbytes > 126e6 else "outputs fit in L2"}
        if label == "mask_build":
            qs = bm.q_side()
            cq = bsmt._BlockMaskQ()
            cq.q_num_blocks = qs["q_num_blocks"].data_ptr()
            cq.q_indices = qs["q_indices"].data_ptr()
            cq.full_q_num_blocks = qs["full_q_num_blocks"].data_ptr()
            cq.full_q_indices = qs["full_q_indices"].data_ptr()
            c = bm._c()
            ms = _time_launches(lambda: bsmt._lib.bsmt_block_mask_transpose(
                ctypes.byref(c), ctypes.byref(cq), ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)))
            qbytes = 2 * 4 * Bm * Hm * KB + 2 * 4 * Bm * Hm * KB * QB
            gbs = qbytes / (ms * 1e-3) / 1e9
            res["q_side_transpose"] = {"ms": ms, "bytes": qbytes, "achieved_gbs": gbs, "peak_gbs": hbm_peak,
                                       "frac": gbs / hbm_peak}
        bsmt.check_device_status(dev)
    # split-KV on a decode-like shape: one q-block per head over a long kv
    # cache, no mask (every tile computed), plain path vs 8 slices
    Bd, Hqd, Hkvd, Md, Nd, Dd, S = 1, 32, 8, 128, 32768, 128, 8
    g = torch.Generator(device="cpu").manual_seed(7)
    qd, kd, vd = (torch.randn(shape, generator=g).to(torch.bfloat16).to(dev)
                  for shape in ((Bd, Hqd, Md, Dd), (Bd, Hkvd, Nd, Dd), (Bd, Hkvd, Nd, Dd)))
    out = torch.empty((Bd, Hqd, Md, Dd), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((Bd, Hqd, Md), dtype=torch.float32, device=dev)
    ws = torch.empty(bsmt.splitkv_workspace_bytes(Bd, Hqd, Md, Dd, S), dtype=torch.uint8, device=dev)
    flops = Bd * Hqd * ((Md + 127) // 128) * ((Nd + 127) // 128) * 4 * 128 * 128 * Dd
    ms1 = _time_launches(lambda: bsmt.flex_attention(qd, kd, vd, enable_gqa=True, out=out, lse=lse), reps=5)
    mss = _time_launches(lambda: bsmt.flex_attention(qd, kd, vd, enable_gqa=True, out=out, lse=lse,
                                                     num_splits=S, workspace=ws), reps=5)
    bsmt.check_device_status(dev)
    # varlen: the packed-document workload in the cu_seqlens form (tokens, H, D)
    lens = workloads.document_lengths(16384, workloads.get(4).seed)
    cu = torch.tensor([0] + list(np.cumsum(lens)), dtype=torch.int32, device=dev)
    T, Hv = int(sum(lens)), 32
    qv, kv_, vv = (torch.randn((T, Hv, 128), generator=g).to(torch.bfloat16).to(dev) for _ in range(3))
    ids = bsmt.seqlens_to_doc_ids(cu, T)
    bmv = bsmt.create_block_mask(bsmt.and_masks(bsmt.document(ids), bsmt.causal()), 1, 1, T, T, device=dev)
    vflops = counted_flops(bmv, 128) * Hv
    msv = _time_launches(lambda: bsmt.flex_attention_varlen(qv, kv_, vv, cu, cu, causal=True), reps=5)
    bsmt.check_device_status(dev)
    res["varlen_doc_causal"] = {"shape": f"{len(lens)} packed sequences, {T} tokens, H=32, D=128, causal",
                                "ms": msv, "tflops": vflops / (msv * 1e-3) / 1e12,
                                "note": "includes doc-id and block-mask kernels per call"}
    # the same forward kernel on long rows of full tiles (no mask) and causal
    long_rows = []
    for (Bl, Hl, Sl, Dl, causal_l) in ((1, 32, 8192, 128, False), (1, 32, 8192, 128, True)):
        ql, kl, vl = (torch.randn((Bl, Hl, Sl, Dl), generator=g).to(torch.bfloat16).to(dev) for _ in range(3))
        bml = bsmt.create_block_mask(bsmt.causal(), Bl, Hl, Sl, Sl, device=dev) if causal_l else None
        tiles = (int(bml.kv_num_blocks.sum()) + int(bml.full_kv_num_blocks.sum())) if causal_l \
            else Bl * Hl * ((Sl + 127) // 128) ** 2
        msl = _time_launches(lambda: bsmt.flex_attention(ql, kl, vl, block_mask=bml), reps=5)
        long_rows.append({"shape": f"B={Bl} H={Hl} S={Sl} D={Dl}", "mask": "causal" if causal_l else "none",
                          "ms": msl, "tflops": tiles * 4 * 128 * 128 * Dl / (msl * 1e-3) / 1e12})
        del ql, kl, vl
    bsmt.check_device_status(dev)
    res["long_rows"] = long_rows
    res["splitkv_decode"] = {"shape": f"B={Bd} Hq={Hqd} Hkv={Hkvd} M={Md} N={Nd} D={Dd}, no mask", "splits": S,
                             "plain_ms": ms1, "plain_tflops": flops / (ms1 * 1e-3) / 1e12,
                             "split_ms": mss, "split_tflops": flops / (mss * 1e-3) / 1e12}
    return res


def workload_sweep(bsmt, dev, peak_tflops: float, hbm_peak: float) -> list:
    """Each of the five workloads on its own: the attention kernel alone (CUDA
    graph of repeated launches, CUDA events), its counted TFLOP/s and fraction
    of the measured bf16 peak, the builder at the workload's own shape (GB/s of
    its four outputs) and the sparsity."""
    res = []
    for w in workloads.WORKLOADS:
        data = workloads.make(w)
        q, k, v = (t.to(dev) for t in (data["q"], data["k"], data["v"]))
        mask = bsmt.mask_from_tree(data["mask"], device=dev)
        mods = [bsmt.ScoreMod(m.kind, m.value, None if m.slopes is None else m.slopes.to(dev))
                for m in bsmt.score_mods_from_list(data["score_mods"])]
        bm = bsmt.create_block_mask(mask, w.B, w.Hq, w.M, w.N, device=dev)
        out = torch.empty((w.B, w.Hq, w.M, w.D), dtype=torch.bfloat16, device=dev)
        lse = torch.empty((w.B, w.Hq, w.M), dtype=torch.float32, device=dev)
        reps = 20 if w.index <= 2 else 5
        ms = _time_launches(lambda: bsmt.flex_attention(q, k, v, block_mask=bm, score_mod=mods, scale=w.scale,
                                                        enable_gqa=w.enable_gqa, out=out, lse=lse), reps=reps)
        ms_b = _time_launches(lambda: bsmt.create_block_mask(mask, w.B, w.Hq, w.M, w.N, device=dev, out=bm),
                              reps=20)
        bsmt.check_device_status(dev)
        flops = counted_flops(bm, w.D)
        tf = flops / (ms * 1e-3) / 1e12
        Bm, Hm, QB, KB = bm.shape
        nbytes = 2 * 4 * Bm * Hm * QB + 2 * 4 * Bm * Hm * QB * KB
        qkv_bytes = sum(x.numel() * 2 for x in (q, k, v))
        res.append({"index": w.index, "workload": w.name, "attn_ms": ms, "counted_gflop": flops / 1e9,
                    "tflops": tf, "frac": tf / peak_tflops, "frac_of_datasheet": tf / DATASHEET_BF16_TFLOPS,
                    "builder_ms": ms_b, "builder_gbs": nbytes / (ms_b * 1e-3) / 1e9,
                    "builder_frac": nbytes / (ms_b * 1e-3) / 1e9 / hbm_peak,
                    "sparsity_pct": bm.sparsity(),
                    "l2": "inputs larger than L2" if qkv_bytes > 126e6 else "inputs fit in L2 (repeated launches)"})
        del q, k, v, out, lse, bm
    torch.cuda.empty_cache()
    return res


def all_partial(bsmt, bm):
    """The same kept tiles as ``bm``, every one listed as PARTIAL (no FULL
    list): the kernel then applies mask_mod on every tile. Built from the
    block-level dense map (the library's to_dense kernel); each row's kept kv
    blocks in ascending order, then zeros."""
    dense = bm.to_dense()
    KB = dense.shape[-1]
    ar = torch.arange(KB, dtype=torch.int32, device=dense.device)
    key = torch.where(dense > 0, ar, ar + KB)
    idx = torch.sort(key, dim=-1).values
    num = dense.sum(-1, dtype=torch.int32)
    idx = torch.where(ar < num[..., None], idx, torch.zeros_like(idx)).to(torch.int32).contiguous()
    return bsmt.BlockMask.from_kv_blocks(num.contiguous(), idx, torch.zeros_like(num), torch.zeros_like(idx),
                                         mask_mod=bm.mask_mod, seq_lengths=bm.seq_lengths)


def full_partial_ablation(bsmt, dev) -> list:
    """The tensorplay.nn.attention page (BlockMask "Details" item 2) stores
    full blocks apart so that mask_mod is skipped on them. Each case is timed
    with its BlockMask and with every kept tile listed as partial (same tiles,
    same output bits)."""
    res = []
    g = torch.Generator(device="cpu").manual_seed(11)
    w5 = workloads.get(5)
    d5 = workloads.make(w5)
    cases = [(w5.name, d5["q"], d5["k"], d5["v"], d5["mask"], w5.enable_gqa),
             ("causal_b1_h32_s8192_d128",) + tuple(torch.randn((1, 32, 8192, 128), generator=g).to(torch.bfloat16)
                                                   for _ in range(3)) + (("causal",), False)]
    for name, qh, kh, vh, tree, gqa in cases:
        q, k, v = (t.to(dev) for t in (qh, kh, vh))
        B, Hq, M, D = q.shape
        N = k.shape[2]
        mask = bsmt.mask_from_tree(tree, device=dev)
        bm = bsmt.create_block_mask(mask, B, Hq, M, N, device=dev)
        bmp = all_partial(bsmt, bm)
        outs = []
        times = []
        for b in (bm, bmp):
            out = torch.empty((B, Hq, M, D), dtype=torch.bfloat16, device=dev)
            lse = torch.empty((B, Hq, M), dtype=torch.float32, device=dev)
            times.append(_time_launches(lambda: bsmt.flex_attention(q, k, v, block_mask=b, enable_gqa=gqa, out=out,
                                                                    lse=lse), reps=5))
            outs.append((out, lse))
        bsmt.check_device_status(dev)
        flops = counted_flops(bm, D)
        res.append({"case": name, "full_and_partial_ms": times[0], "all_partial_ms": times[1],
                    "full_and_partial_tflops": flops / (times[0] * 1e-3) / 1e12,
                    "all_partial_tflops": flops / (times[1] * 1e-3) / 1e12,
                    "speedup": times[1] / times[0],
                    "full_tiles": int(bm.full_kv_num_blocks.sum()), "partial_tiles": int(bm.kv_num_blocks.sum()),
                    "outputs_identical": bool(torch.equal(outs[0][0], outs[1][0]) and
                                              torch.equal(outs[0][1], outs[1][1]))})
        del q, k, v, outs
    torch.cuda.empty_cache()
    return res


def counted_flops(bm, D: int) -> int:
    """4*128*128*D per kept tile per (b, hq); the mask is built at [B, Hq]."""
    tiles = int(bm.kv_num_blocks.sum().item()) + int(bm.full_kv_num_blocks.sum().item())
    return tiles * 4 * 128 * 128 * D


def run_builder_only(bsmt, args, w):
    """The block-mask builder alone: --steps launches at (B, H) of the workload
    (or --batch / --heads), timed through a CUDA graph. Bytes are the four
    output tensors (and the document ids read, if any)."""
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    data = workloads.make(w)
    mask = bsmt.mask_from_tree(data["mask"], device=dev)
    H = args.heads or w.Hq
    bm = bsmt.create_block_mask(mask, w.B, H, w.M, w.N, device=dev)
    ms = _time_launches(lambda: bsmt.create_block_mask(mask, w.B, H, w.M, w.N, device=dev, out=bm),
                        reps=max(1, args.steps))
    bsmt.check_device_status(dev)
    Bm, Hm, QB, KB = bm.shape
    nbytes = 2 * 4 * Bm * Hm * QB + 2 * 4 * Bm * Hm * QB * KB
    peaks, _ = load_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    print(json.dumps({"workload": w.name, "B": Bm, "H": Hm, "ms": ms, "bytes": nbytes,
                      "achieved_gbs": nbytes / (ms * 1e-3) / 1e9, "frac_of_hbm": nbytes / (ms * 1e-3) / 1e9 / hbm}))


# ------------------------------------------------------------------ oracle
def cpu_baseline(w, data, max_rows: int = 16384, chunk: int = 1024, cls=None):
    """The fp64 oracle, as it stands, on a bounded sample of the workload: whole
    q-blocks of (b=0, hq=0) from the top of the sequence (the rows with the most
    kept tiles), in chunks of ``chunk`` rows, counted with the same tile rule as
    the GPU metric."""
    from threadpoolctl import threadpool_info, threadpool_limits
    from oracle import attention as oa
    # the oracle's matrix products use one BLAS thread per host core given to this process
    threadpool_limits(len(os.sched_getaffinity(0)))
    from oracle import block_mask as obm

    rows_per_block = 128
    QB = (w.M + 127) // 128
    nblk = max(1, min(QB, max_rows // rows_per_block))
    qbs = list(range(QB - nblk, QB))
    samples = [(0, 0, qb * 128 + r) for qb in qbs for r in range(128) if qb * 128 + r < w.M]
    block_mask = None
    if cls is None:
        # The oracle's block mask on its own: one (b, h) slice with B = H = 1 (the
        # workloads' masks do not depend on the head), classification and
        # compaction; GB/s of its four outputs, as for the GPU builder.
        t0 = time.perf_counter()
        bmo = obm.create_block_mask(data["mask"], 1, 1, w.M, w.N)
        t_bm = time.perf_counter() - t0
        nbytes = sum(int(a.nbytes) for a in bmo.values())
        cls = bmo["kv_num_blocks"][0, 0] + bmo["full_kv_num_blocks"][0, 0]  # kept tiles per q-block row
        block_mask = {"value": nbytes / t_bm / 1e9, "unit": "GB/s", "seconds": t_bm,
                      "sample": f"create_block_mask of one (b, h) slice: {QB} x {(w.N + 127) // 128} tiles, "
                                f"{nbytes} bytes of outputs, one core"}
        tiles = sum(int(cls[qb]) for qb in qbs)
    else:
        tiles = sum(int((cls[qb] > 0).sum()) for qb in qbs)
    flops = tiles * 4 * 128 * 128 * w.D
    t0 = time.perf_counter()
    for c0 in range(0, len(samples), chunk):
        oa.flex_attention_sampled(data["q"], data["k"], data["v"], samples[c0:c0 + chunk], data["mask"],
                                  data["score_mods"], w.scale, w.enable_gqa)
    dt = time.perf_counter() - t0
    blas = max([p.get("num_threads", 1) for p in threadpool_info()] or [1])
    res = {"value": flops / dt / 1e12, "unit": UNIT, "cores": len(os.sched_getaffinity(0)), "blas_threads": int(blas),
           "kind": "oracle",
           "sample": f"{len(samples)} query rows = q-blocks {qbs[0]}..{qbs[-1]} of (b=0, hq=0), "
                     f"{tiles} kept tiles, {dt:.1f} s"}
    if block_mask is not None:
        res["block_mask"] = block_mask
    return res


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from oracle import block_mask as obm
    data = workloads.make(w)
    cls = obm.tile_classes(data["mask"], 0, w.M, w.N)   # counting only, outside the timed oracle calls
    base = None
    times = []
    total = args.warmup + args.steps
    for i in range(total):
        r = cpu_baseline(w, data, max_rows=1024, cls=cls)
        if i >= args.warmup:
            times.append(r)
        base = r
    vals = [t["value"] for t in times]
    value = statistics.mean(vals) if vals else 0.0
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "seq_len": w.M, "D": w.D},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": base["cores"], "kind": "oracle",
                         "sample": "each step: " + base["sample"]},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# -------------------------------------------------------------------- GPU
def main():
    args = parse()
    w = workloads.get(args.workload)
    if args.batch:
        import dataclasses
        w = dataclasses.replace(w, B=args.batch)
    if args.impl == "reference":
        run_reference(args, w)
        return

    import block_sparse_masked_tile_b200 as bsmt

    if args.builder_only:
        run_builder_only(bsmt, args, w)
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)

    data = workloads.make(w, seed_offset=rank)
    q, k, v = (t.to(dev) for t in (data["q"], data["k"], data["v"]))
    mask = bsmt.mask_from_tree(data["mask"], device=dev)
    mods = bsmt.score_mods_from_list(data["score_mods"])
    bm = bsmt.create_block_mask(mask, w.B, w.Hq, w.M, w.N, device=dev)
    out = torch.empty((w.B, w.Hq, w.M, w.D), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.B, w.Hq, w.M), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(attn_events=None):
        bsmt.create_block_mask(mask, w.B, w.Hq, w.M, w.N, device=dev, out=bm)
        if attn_events is not None:
            attn_events[0].record(stream)
        bsmt.flex_attention(q, k, v, block_mask=bm, score_mod=mods, scale=w.scale, enable_gqa=w.enable_gqa,
                            out=out, lse=lse)
        if attn_events is not None:
            attn_events[1].record(stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(dev)
    bsmt.check_device_status(dev)
    flops = counted_flops(bm, w.D)
    sparsity = bm.sparsity()
    if args.backward_only:
        r = time_backward(bsmt, w, q, k, v, out, lse, bm, mods, dev, flops, reps=max(1, args.steps))
        if rank == 0:
            print(json.dumps({"workload": w.name, "B": w.B, "backward": r}), flush=True)
        if dist:
            dist.destroy_process_group()
        return

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        clk.mark_start()
        start.record(stream)
        for i in range(args.steps):
            step(ev[i])
        end.record(stream)
        torch.cuda.synchronize(dev)
        clk.mark_end()
    if dist:
        dist.barrier()
    bsmt.check_device_status(dev)
    ms = start.elapsed_time(end) / args.steps
    attn_ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    (ms, attn_ms), total_flops = reduce_over_ranks(dist, dev, (ms, attn_ms), flops)
    value = total_flops / (ms * 1e-3) / 1e12

    # end to end through the public API with host buffers
    hq_, hk_, hv_ = (x.pin_memory() for x in (data["q"], data["k"], data["v"]))
    ho = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    hl = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
    # the mask with its document ids (if any) in pinned host memory, and ALiBi
    # slopes on the host: the host-buffer call copies them in itself
    hmask = bsmt.mask_from_tree(data["mask"])
    doc_host = []
    if hmask.q_doc_ids is not None:
        doc_host = [hmask.q_doc_ids.pin_memory(), hmask.kv_doc_ids.pin_memory()]
        hmask = bsmt.MaskMod(hmask.nodes, doc_host[0], doc_host[1])
    hmods = bsmt.score_mods_from_list(data["score_mods"])
    slopes_host = [m.slopes for m in hmods if m.slopes is not None]
    hws = torch.empty(bsmt.host_workspace_bytes(w.B, w.Hq, w.Hkv, w.M, w.N, w.D, hmask), dtype=torch.uint8,
                      device=dev)

    def e2e_step():
        # the public host-buffer call (bsmt_flex_attention_host): document ids
        # and slopes in, block mask built on the device, pieces' copies in and
        # out pipelined with their attention; returns once out/lse are on the host
        bsmt.flex_attention_host(hq_, hk_, hv_, mask_mod=hmask, score_mod=hmods, scale=w.scale,
                                 enable_gqa=w.enable_gqa, device=dev, out=ho, lse=hl, workspace=hws)

    e2e_step()
    if dist:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for _ in range(args.e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1) / args.e2e_steps
    (e2e_ms,), _ = reduce_over_ranks(dist, dev, (e2e_ms,), 0)
    h2d = (sum(x.numel() * x.element_size() for x in (hq_, hk_, hv_)) + sum(x.numel() * 4 for x in doc_host)
           + sum(x.numel() * 4 for x in slopes_host))
    d2h = ho.numel() * ho.element_size() + hl.numel() * hl.element_size()

    peaks, peak_src = load_peaks()
    hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    side = None if args.no_side_kernels else side_kernels(bsmt, mask, w, dev, hbm_peak)
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    sustained = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    clocks = clk.summary()
    # a timed region long enough for the 1 kW power cap to act runs at the
    # sustained matmul rate, so it is held against the sustained peak
    capped = bool(clocks.get("in_window")) and "sw_power_cap" in clocks["reasons"]
    peak = sustained if capped else burst
    if side is not None:
        side["backward"] = time_backward(bsmt, w, q, k, v, out, lse, bm, mods, dev, flops)
        side["workloads"] = workload_sweep(bsmt, dev, burst, hbm_peak)
        side["full_partial_ablation"] = full_partial_ablation(bsmt, dev)
    attn_tflops = (flops / (attn_ms * 1e-3)) / 1e12
    prof = profile_figures(w.name)
    line = {
        "metric": METRIC,
        "value": value,
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": max(3, args.warmup),
        "ms_per_step": ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {
            "workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "seq_len": w.M, "D": w.D,
            "mask": data["mask"][0] if w.mask != "doc_causal" else "document and causal",
            "counted_gflop_per_gpu_step": flops / 1e9, "sparsity_pct": sparsity,
            "l2": "inputs larger than L2 (q+k+v = %.0f MB per step); L2 not flushed" % (
                sum(x.numel() * 2 for x in (q, k, v)) / 1e6),
            "parallelism": f"dp{world} (independent batches per GPU)",
        },
        "roofline": {
            "bound": "tensor",
            "achieved": attn_tflops,
            "peak": peak,
            "unit": "TFLOP/s",
            "frac": attn_tflops / peak,
            "traffic": prof["traffic"],
            "kernel": "attn_fwd_kernel",
            # the ncu capture's pipe shares (of active cycles) for the same source;
            # MUFU shows how close the exponentials are to bounding the kernel
            "tensor_pipe_pct": prof["tensor_pipe_pct"],
            "mufu_pipe_pct": prof["mufu_pipe_pct"],
            "peak_source": (f"{peak_src} bf16_tflops_sustained (sw_power_cap active in the timed region); burst "
                            f"{burst}; datasheet {DATASHEET_BF16_TFLOPS}") if capped else
                           (f"{peak_src} bf16_tflops (burst: no power cap in the timed region); sustained "
                            f"{sustained}; datasheet {DATASHEET_BF16_TFLOPS}"),
            "frac_of_datasheet": attn_tflops / DATASHEET_BF16_TFLOPS,
            "attn_ms": attn_ms,
        },
        "e2e": {"value": total_flops / (e2e_ms * 1e-3) / 1e12, "unit": UNIT,
                "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "ms_per_step": e2e_ms},
        "side_kernels": side,
        # each timed step is one builder launch and one attention launch (the
        # committed launch list of this command shows exactly these)
        "gpu_launches": 2 * args.steps,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, data)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
