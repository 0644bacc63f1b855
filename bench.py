"""Benchmark of the RLT hot path on B200: one step = the encoder prefill of a
batch of sequences plus every recurrent decoder transition of that batch (all
positions, prompt and response, no reset), through the C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference] [--all-workloads]

Prints one JSON line (rank 0). N > 1 runs under torchrun: every rank runs the
whole workload on its own GPU (sequences are independent, no collective on the
data path); the reported time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from token_recurrent_decoding_b200 import configs, inputs, ranks, roofline  # noqa: E402

METRIC = "decoder sequence-steps/s (bf16, B200) and % of step roofline (HBM/tensor)"
DEFAULT_WORKLOAD = "m140_bf16"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
WORKLOAD_TEXT = {
    "tiny_fp32": "tiny fp32 RLT d=64 4x16 heads, 2+2 layers, W=8, G=1; B=2 x T=64",
    "m50_bf16": "~50M RLT bf16 d=512 8x64, 6+6, FFN 2048, W=64, G=1, alpha=1; B=64 x T=1024",
    "m50_bf16_alpha0": "~50M RLT bf16 as m50_bf16 with alpha=0 (feedback off); B=64 x T=1024",
    "m140_bf16": ("~140M RLT bf16 d=768 12x64, 12+12, FFN 3072, W=128, G=L_D, alpha=1; "
                  "B=256 x T=1024 (prompt 768 + 256 response steps, no reset)"),
    "tied_bf16": ("tied RLT bf16 48+48 shared attention/FFN, d=2048 16x128, SwiGLU 5632, "
                  "W=256, G=1; B=32 x (3072 prompt + 1024 response) = 4096 steps"),
    "ragged_bf16": ("ragged ~140M RLT bf16 G=1, 1024 sequences, prompt U[128,2048] + 256 "
                    "response steps; ready-set scheduler"),
}


# DRAM traffic of the dominant kernel from its committed Nsight Compute
# summary: bytes read + written per algorithmic byte, valid only while the
# kernel source hashes to the value recorded with the capture.
ATTN_PROFILE = os.path.join(ROOT, "profiles", "k_attn_decode_bf16_dh64_n256_len512.md")
ATTN_SOURCE = os.path.join(ROOT, "token_recurrent_decoding_b200", "csrc", "attn.cuh")


def attn_traffic_ratio():
    import hashlib
    if not os.path.exists(ATTN_PROFILE):
        return None, "no profile"
    ratio = sha = None
    with open(ATTN_PROFILE) as f:
        for line in f:
            if line.startswith("source sha256"):
                sha = line.split(":", 1)[1].strip().strip("`")
            elif line.startswith("dram bytes per algorithmic byte"):
                ratio = float(line.split(":", 1)[1].strip().strip("`"))
    with open(ATTN_SOURCE, "rb") as f:
        cur = hashlib.sha256(f.read()).hexdigest()
    if ratio is None or sha != cur:
        return None, "kernel changed since the capture" if ratio is not None else "no ratio"
    return ratio, os.path.relpath(ATTN_PROFILE, ROOT)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ ranks
def dist_setup(n_gpus):
    import torch
    if n_gpus <= 1 or "RANK" not in os.environ:
        return 0, 1, None
    import datetime
    import torch.distributed as dist
    local = int(os.environ.get("LOCAL_RANK", 0))
    torch.cuda.set_device(local)
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    return dist.get_rank(), dist.get_world_size(), dist


def max_over_ranks(x: float, dist) -> float:
    return ranks.max_over_ranks(x, dist, device="cuda")


def barrier(dist):
    if dist is not None:
        dist.barrier()


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi sampled every 200 ms while the timed region runs."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        # raw samples (the JSON line carries their summary); RLT_CLOCKS_DIR keeps them
        import tempfile
        out = os.environ.get("RLT_CLOCKS_DIR") or tempfile.gettempdir()
        self.path = os.path.join(out, f"clocks_bench_{os.getpid()}.csv")

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", str(self.gpu)], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() in ("active", "1"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ our arm
class Runner:
    """Owns the device model and the seeded inputs of one workload."""

    def __init__(self, wl, device="cuda", rank=0, world=1):
        import torch
        from token_recurrent_decoding_b200.rlt import Model
        self.torch = torch
        self.wl = wl
        cfg = wl.model
        self.stream = torch.cuda.Stream()
        w = inputs.make_weights(cfg)
        # weak scaling: the job holds world x B sequences; this rank owns a
        # contiguous shard of them (same lengths, its own tokens)
        lo, hi = ranks.shard_range(world * wl.batch, rank, world)
        self.tok = inputs.make_tokens(cfg.vocab, list(wl.lengths) * world)[lo:hi]
        lengths = np.asarray(wl.lengths, np.int32)
        self.lengths = lengths
        flat = np.concatenate([self.tok[i, :L] for i, L in enumerate(lengths)]).astype(np.int32)
        self.offsets = np.concatenate([[0], np.cumsum(lengths)[:-1]]).astype(np.int32)
        self.ids = np.arange(wl.batch, dtype=np.int32)
        self.tok_dev = torch.from_numpy(flat).to(device)
        self.tok_host = torch.from_numpy(flat).pin_memory()
        self.s_host = torch.empty((wl.batch, cfg.d), dtype=torch.float32).pin_memory()
        self.m = Model(cfg, w, wl.batch, wl.max_len, device=device, stream=self.stream)
        del w
        self.ragged = len(set(wl.lengths)) > 1

    def decode(self):
        if self.ragged:
            self.m.run_ragged(self.ids, self.lengths)
        else:
            self.m.run_sequence(self.ids, int(self.lengths[0]))

    def step(self, ev=None, host=False):
        tok = self.tok_host if host else self.tok_dev
        self.m.prefill_encoder(tok, self.ids, self.offsets, self.lengths)
        if ev is not None:
            ev.record(self.stream)
        self.decode()
        if host:
            self._read_states()

    def time_parallel(self, steps, warmup):
        """Token-parallel decoder pass (feedback-off models, equal lengths):
        encoder prefill, then all positions of every sequence at once; the
        device time of the passes alone."""
        torch = self.torch
        T = int(self.lengths[0])
        ms = []
        for k in range(warmup + steps):
            self.m.prefill_encoder(self.tok_dev, self.ids, self.offsets, self.lengths)
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(self.stream)
            self.m.decoder_parallel(self.ids, T)
            b.record(self.stream)
            torch.cuda.synchronize()
            if k >= warmup:
                ms.append(a.elapsed_time(b))
        return sum(ms) / len(ms)

    def _read_states(self):
        # one d2h copy per sequence of its final s into pinned host memory
        import ctypes as C
        from token_recurrent_decoding_b200 import rlt
        lib = rlt._lib()
        st = C.c_void_p(self.stream.cuda_stream)
        row = self.wl.model.d * 4
        base = self.s_host.data_ptr()
        for i in range(self.wl.batch):
            rc = lib.rlt_get_state(self.m._h, i, C.c_void_p(base + i * row), None, None, st)
            assert rc == 0, rc


def run_ours(args, wl, rank, world, dist, peaks, peaks_src):
    import torch
    r = Runner(wl, rank=rank, world=world)
    st = r.stream
    torch.cuda.synchronize()
    for _ in range(args.warmup):
        r.step()
    torch.cuda.synchronize()
    barrier(dist)

    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
            torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    # the contract numbers are timed with the per-kernel measurement hook off
    r.m.profile(0)
    launches0 = r.m.get_stats()["launches"]
    clk = ClockSampler(torch.cuda.current_device())
    with clk:
        torch.cuda.synchronize()
        barrier(dist)
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(st)
        for k in range(args.steps):
            a, b, c = evs[k]
            a.record(st)
            r.step(ev=b)
            c.record(st)
        t1.record(st)
        torch.cuda.synchronize()
        barrier(dist)
    launches = r.m.get_stats()["launches"] - launches0
    total_ms = t0.elapsed_time(t1)
    enc_ms = sum(a.elapsed_time(b) for a, b, _ in evs)
    dec_ms = sum(b.elapsed_time(c) for _, b, c in evs)
    total_ms = max_over_ranks(total_ms, dist)

    # per-kernel figures from a separate profiled step after the timed region:
    # every profile_stride-th decoder step (and the prefill) replays a graph
    # whose event nodes bracket each kernel, run as one unsplit chain
    torch.cuda.synchronize()
    r.m.profile(args.profile_stride)
    r.step()
    stats = r.m.get_stats()
    r.m.profile(0)

    # end to end through the C ABI with host buffers: tokens from pinned host
    # memory in, every sequence's s_T back into pinned host memory
    e2e_steps = max(1, min(args.steps, 2))
    torch.cuda.synchronize()
    barrier(dist)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(e2e_steps):
        r.step(host=True)
    e1.record(st)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dist) / e2e_steps

    cfg = wl.model
    seq_steps = wl.seq_steps
    value = world * seq_steps * args.steps / (total_ms / 1e3)
    hbm = peaks["hbm_gbs"]
    tc = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    roof = roofline.run_roofline(cfg, wl.lengths, hbm, tc)
    x = stats["xattn"]
    achieved = (x["bytes"] / x["launches"]) / (x["ms"] / x["launches"] / 1e3) / 1e9 if x["launches"] else None
    ratio, traffic_src = attn_traffic_ratio()
    traffic = ratio * x["bytes"] / x["launches"] if (ratio and x["launches"]) else None
    dec_s = dec_ms / 1e3 / args.steps
    enc_s = enc_ms / 1e3 / args.steps
    out = {
        "metric": METRIC,
        "value": value,
        "unit": "seq-steps/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": total_ms / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if cfg.dtype == configs.BF16 else "f32",
        "data": "synthetic (seeded N(0,0.02) weights, uniform tokens)",
        "config": {
            "workload": f"{wl.name}: {WORKLOAD_TEXT.get(wl.name, '')}",
            "batch": wl.batch, "seq_len": wl.max_len, "seq_steps_per_step": seq_steps,
            "window": cfg.window, "mem_groups": cfg.mem_groups,
            "l2": "inputs larger than L2 (no flush): encoder memory %.1f GB" %
                  (cfg.mem_groups * sum(wl.lengths) * 2 * cfg.d *
                   roofline.elem_bytes(cfg) / 1e9),
            "parallelism": f"replicas x{world} (sequences sharded, no data-path collective)",
        },
        "decoder_seq_steps_per_s": world * seq_steps / dec_s,
        "encoder_tokens_per_s": world * seq_steps / enc_s,
        "step_roofline": {
            "decoder_frac": roof["decoder_s"] / dec_s,
            "encoder_frac": roof["encoder_s"] / enc_s,
            "whole_frac": (roof["decoder_s"] + roof["encoder_s"]) / (dec_s + enc_s),
            "decoder_roof_s": roof["decoder_s"], "encoder_roof_s": roof["encoder_s"],
            "peaks": f"{peaks_src}: HBM {hbm} GB/s, bf16 {tc} TFLOP/s (sustained)",
        },
        "roofline": {
            "kernel": "k_attn_decode (decoder cross-attention over M<=t)",
            "bound": "hbm",
            "achieved": achieved,
            "peak": hbm,
            "unit": "GB/s",
            "frac": achieved / hbm if achieved else None,
            "traffic": traffic,
            "traffic_source": traffic_src,
            "algorithmic_bytes_per_launch": (x["bytes"] / x["launches"]) if x["launches"] else None,
            "launches_timed": x["launches"],
            "timing": ("CUDA events around each launch in a profiled step run after the "
                       "contract's timed region (every %d-th decoder step, one chain)"
                       % args.profile_stride),
            "peak_source": peaks_src,
        },
        "kernel_classes": {k: {"ms_profiled": v["ms"],
                               "launches_profiled": v["launches"],
                               "GB_s": (v["bytes"] / (v["ms"] / 1e3) / 1e9) if v["ms"] else None,
                               "TFLOP_s": (v["flops"] / (v["ms"] / 1e3) / 1e12) if v["ms"] else None}
                           for k, v in stats.items() if isinstance(v, dict)},
        "e2e": {"value": world * seq_steps / (e2e_ms / 1e3), "unit": "seq-steps/s",
                "h2d_bytes_per_step": int(r.tok_host.numel() * 4),
                "d2h_bytes_per_step": int(wl.batch * cfg.d * 4)},
        "gpu_launches": int(launches),
        "clocks": clk.summary(),
    }
    if cfg.alpha == 0.0 and not r.ragged:
        # the feedback-off model also runs its decoder token-parallel
        par_ms = max_over_ranks(r.time_parallel(args.steps, 1), dist)
        pr = roofline.decoder_parallel_roofline(cfg, wl.lengths, hbm, tc)
        out["decoder_parallel"] = {
            "seq_steps_per_s": world * seq_steps / (par_ms / 1e3),
            "ms_per_step": par_ms,
            "roofline_s": pr["seconds"],
            "frac": pr["seconds"] / (par_ms / 1e3),
            "TFLOP_s": pr["flops"] / (par_ms / 1e3) / 1e12,
            "bound": "tensor" if pr["flops"] / (tc * 1e12) >= pr["bytes"] / (hbm * 1e9) else "hbm",
        }
    if args.backward and not r.ragged and cfg.dtype == configs.BF16:
        out["backward"] = time_backward(wl, r, dist, hbm, tc)
        if rank == 0 and not args.no_cpu_baseline and "skipped" not in out["backward"]:
            out["backward"]["cpu_baseline"] = cpu_backward_baseline(wl)
    if args.serve and wl.prompt_lengths and not r.ragged and cfg.dtype == configs.BF16:
        out["serve"] = time_serve(wl, r, dist)
    if rank == 0 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(wl, args.cpu_positions)
    return out


def time_backward(wl, r, dist, hbm, tc):
    """Backpropagation through time over the whole workload (outside the
    contract timing): encoder prefill, then one rlt_backward over every
    position of every sequence (recorded forward, reverse traversal, memory
    gradient), upstream gradients dL/ds_t seeded N(0, 1); one short call first
    warms the graphs and tensor maps. Reports seq-steps/s of the timed call."""
    import torch
    cfg = wl.model
    T = int(r.lengths[0])
    m = r.m
    need = m.backward_workspace_bytes(wl.batch, T)
    free, _ = torch.cuda.mem_get_info()
    if need + 3 * wl.batch * wl.max_len * cfg.d * 4 > 0.9 * free:
        return {"skipped": "workspace %.1f GB for %d x %d positions exceeds free device memory "
                           "%.1f GB (chunked backpropagation through rlt_backward's carried "
                           "gradient covers such runs)" % (need / 1e9, wl.batch, T, free / 1e9)}
    g = torch.Generator(device="cuda").manual_seed(2)
    sgrad = torch.randn((wl.batch, T, cfg.d), generator=g, device="cuda")
    grads = {k: torch.zeros(v, device="cuda") for k, v in m.grad_shapes().items()}
    egrad = torch.zeros((wl.batch, wl.max_len, cfg.d), device="cuda")
    ws = torch.empty(m.backward_workspace_bytes(wl.batch, T), dtype=torch.uint8, device="cuda")
    ids = r.ids
    m.prefill_encoder(r.tok_dev, ids, r.offsets, r.lengths)
    m.backward(ids, sgrad[:, :8].contiguous(), grads=grads, egrad=egrad, workspace=ws)
    m.prefill_encoder(r.tok_dev, ids, r.offsets, r.lengths)
    torch.cuda.synchronize()
    barrier(dist)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(r.stream)
    m.backward(ids, sgrad, grads=grads, egrad=egrad, workspace=ws)
    b.record(r.stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(b), dist)
    assert m.poll_device_error() == 0
    finite = bool(torch.isfinite(grads["dec.0.wqkv"]).all().item())
    gb = ws.numel() / 1e9
    del ws, grads, egrad, sgrad
    torch.cuda.empty_cache()
    world = dist.get_world_size() if dist is not None else 1
    br = roofline.backward_roofline(cfg, wl.lengths, hbm, tc)
    return {"seq_steps_per_s": world * wl.batch * T / (ms / 1e3), "ms_per_pass": ms,
            "roofline_s": br["seconds"], "frac": br["seconds"] / (ms / 1e3),
            "TFLOP_s": br["flops"] / (ms / 1e3) / 1e12, "workspace_gb": gb,
            "grads_finite": finite,
            "note": "rlt_backward over all positions: recorded forward on the step kernels, "
                    "reverse traversal, memory-row gradient and projection"}


def time_serve(wl, r, dist):
    """The autoregressive form of the workload (outside the contract timing):
    prefill the prompts only, run the decoder over them, then generate the
    response tokens with rlt_serve_step (transition, next-token head,
    temperature-1 draw from seeded uniforms, encoder append) on a model that
    keeps the encoder cache. Reports generated tokens per second."""
    import torch
    from token_recurrent_decoding_b200.rlt import Model
    cfg = wl.model
    P = int(wl.prompt_lengths[0])
    G = wl.max_len - P
    w = inputs.make_weights(cfg)
    m = Model(cfg, w, wl.batch, wl.max_len, stream=r.stream, enc_cache=True)
    del w
    r.m.close()  # the contract model and its arena are no longer needed
    r.m.arena = None
    torch.cuda.empty_cache()
    tok = r.tok[:, :P]
    flat = torch.from_numpy(np.ascontiguousarray(tok).reshape(-1).astype(np.int32)).cuda()
    ids = np.arange(wl.batch, dtype=np.int32)
    m.prefill_encoder(flat, ids, ids * P, [P] * wl.batch)
    m.run_sequence(ids, P - 1)
    g = torch.Generator(device="cuda").manual_seed(1)
    uni = torch.rand((G, wl.batch), generator=g, device="cuda")
    logits = torch.empty((wl.batch, cfg.vocab), dtype=torch.float32, device="cuda")
    out = torch.empty(wl.batch, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    barrier(dist)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(r.stream)
    for k in range(G):
        m.serve_step(ids, 1.0, uni[k], logits, out)
    b.record(r.stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(b), dist)
    assert m.poll_device_error() == 0
    m.close()
    world = dist.get_world_size() if dist is not None else 1
    return {"generated_tokens_per_s": world * wl.batch * G / (ms / 1e3), "ms_per_token_step": ms / G,
            "sequences": wl.batch, "prompt": P, "generated": G,
            "note": "prompt prefill + decoder over the prompt, then rlt_serve_step per token "
                    "(transition, head E s_t, temperature-1 draw, encoder append)"}


# ------------------------------------------------------------------ oracle arm
def cpu_sample(wl, positions):
    cores = os.cpu_count() or 1
    nseq = min(wl.batch, max(1, cores))
    lens = [min(positions, L) for L in wl.lengths[:nseq]]
    return nseq, lens, cores


def cpu_baseline(wl, positions):
    """The fp32 oracle as it stands, on the host cores, over a bounded sample:
    the first `positions` tokens of `cores` sequences (encoder + decoder)."""
    import oracle
    nseq, lens, cores = cpu_sample(wl, positions)
    cfg = wl.model
    w = inputs.make_weights(cfg)
    o = oracle.Oracle(cfg, w, "f32")
    tok = inputs.make_tokens(cfg.vocab, wl.lengths)[:nseq]
    t = time.perf_counter()
    _, used = o.run_batch(tok, lens, n_threads=cores)
    dt = time.perf_counter() - t
    return {"value": sum(lens) / dt, "unit": "seq-steps/s", "cores": used, "kind": "oracle",
            "sample": f"{nseq} sequences x first {lens[0]} positions (encoder + decoder, fp32 "
                      f"oracle, OpenMP over sequences), {dt:.1f} s"}


def cpu_backward_baseline(wl, positions=8):
    """The gradient oracle (float64 restatement differentiated by
    torch.autograd) as it stands, on the host cores, over a bounded sample:
    one sequence's first `positions` positions from s*, its encoder output
    from the C oracle."""
    import torch

    import oracle
    from oracle import bptt
    cfg = wl.model
    w = inputs.make_weights(cfg)
    tok = inputs.make_tokens(cfg.vocab, wl.lengths)[0, :positions]
    e, _ = oracle.Oracle(cfg, w).encode(tok)
    G = np.random.default_rng(3).standard_normal((positions, cfg.d))
    win0 = np.zeros((cfg.n_dec, 2, max(cfg.window - 1, 0), cfg.d))
    t = time.perf_counter()
    bptt.chunk_grads(cfg, w, e, w["sstar"], win0, 0, positions, G)
    dt = time.perf_counter() - t
    return {"value": positions / dt, "unit": "seq-steps/s", "cores": torch.get_num_threads(),
            "kind": "oracle",
            "sample": f"1 sequence x first {positions} positions (gradient oracle: float64 "
                      f"torch autograd over the decoder), {dt:.1f} s"}


def run_reference(args, wl, rank, world):
    if rank != 0:
        return None
    import oracle
    cfg = wl.model
    nseq, lens, cores = cpu_sample(wl, args.cpu_positions)
    w = inputs.make_weights(cfg)
    o = oracle.Oracle(cfg, w, "f32")
    tok = inputs.make_tokens(cfg.vocab, wl.lengths)[:nseq]
    for _ in range(args.warmup):
        o.run_batch(tok, [1] * nseq, n_threads=cores)
    t = time.perf_counter()
    used = 1
    for _ in range(args.steps):
        _, used = o.run_batch(tok, lens, n_threads=cores)
    dt = time.perf_counter() - t
    value = sum(lens) * args.steps / dt
    sample = (f"{nseq} sequences x first {lens[0]} positions per step (encoder + decoder, "
              f"fp32 oracle, OpenMP over sequences)")
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "seq-steps/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt * 1e3 / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": f"{wl.name}: {WORKLOAD_TEXT.get(wl.name, '')}",
                   "batch": wl.batch, "seq_len": wl.max_len},
        "cpu_baseline": {"value": value, "unit": "seq-steps/s", "cores": used, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "seq-steps/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=list(configs.workloads()))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--all-workloads", action="store_true",
                    help="one JSON line per workload (not the default contract line)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--serve", action=argparse.BooleanOptionalAction, default=True,
                    help="also time the autoregressive form (generated tokens/s)")
    ap.add_argument("--backward", action=argparse.BooleanOptionalAction, default=True,
                    help="also time backpropagation through time over the workload")
    ap.add_argument("--cpu-positions", type=int, default=24)
    ap.add_argument("--profile-stride", type=int, default=64,
                    help="event-time every k-th decoder step for the per-kernel roofline")
    args = ap.parse_args()

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", 0))
        out = run_reference(args, configs.workloads()[args.workload], rank, args.gpus)
        if out is not None:
            print(json.dumps(out), flush=True)
        return

    import torch
    rank, world, dist = dist_setup(args.gpus)
    peaks, src = load_peaks()
    names = list(configs.workloads()) if args.all_workloads else [args.workload]
    try:
        for name in names:
            out = run_ours(args, configs.workloads()[name], rank, world, dist, peaks, src)
            if rank == 0:
                print(json.dumps(out), flush=True)
            torch.cuda.empty_cache()
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
