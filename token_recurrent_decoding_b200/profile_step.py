"""Short runs of the hot path for profilers (few launches, device-timed).

Decoder steps at a chosen position:

    python -m token_recurrent_decoding_b200.profile_step --workload m140_bf16 --t 512 --steps 2

prefills the encoder for the batch (--kernel picks the persistent one-launch
step or the chain of kernels; --max-len shrinks the sequence length and
so the arena), places every sequence at position t with a
random state imported through rlt_set_state (s and the window of every layer),
and runs `steps` decoder steps with direct launches on the legacy stream, so a
profiler sees each kernel once per layer per step. With --graph the steps run
on a side stream instead, i.e. through the captured step graphs (two chains
for large batches, programmatic dependent launch between kernels), as a
serving loop would; the first step captures. Prints the CUDA-event time of
each step and its algorithmic bytes.

The decode attention kernel alone, through rlt_attend:

    python -m token_recurrent_decoding_b200.profile_step --attend --n 256 --heads 12 \
        --dh 64 --cap 1024 --len 1024 --reps 3
"""
from __future__ import annotations

import argparse
import json

import numpy as np


def run_steps(args):
    import torch

    from . import configs, inputs, roofline
    from .rlt import Model
    wl = configs.workloads()[args.workload]
    cfg = wl.model
    if args.layers:  # same shapes, fewer blocks (a profiler's device memory stays small)
        cfg = cfg.replace(n_enc=args.layers, n_dec=args.layers,
                          mem_groups=1 if cfg.mem_groups == 1 else args.layers)
    B = args.batch or wl.batch
    T = args.max_len or wl.max_len
    if args.t + args.steps > T:
        raise SystemExit(f"--t {args.t} + --steps {args.steps} exceeds the sequence length {T}")
    lengths = [T] * B
    w = inputs.make_weights(cfg)
    tok = inputs.make_tokens(cfg.vocab, lengths)
    m = Model(cfg, w, B, T)
    del w
    if args.kernel:
        from . import rlt
        m.set_step_kernel(rlt.STEP_FUSED if args.kernel == "fused" else rlt.STEP_CHAIN)
    flat = torch.from_numpy(tok.reshape(-1).astype(np.int32)).cuda()
    offsets = np.arange(B, dtype=np.int32) * T
    m.prefill_encoder(flat, list(range(B)), offsets, lengths)
    g = torch.Generator(device="cuda").manual_seed(5)
    s = torch.randn(cfg.d, generator=g, device="cuda")
    cache = torch.randn((cfg.n_dec, 2, max(cfg.window - 1, 0), cfg.d), generator=g,
                        device="cuda").to(m.wdtype)
    for i in range(B):
        m.set_state(i, s, cache, args.t)
    torch.cuda.synchronize()
    ids = list(range(B))
    st = torch.cuda.Stream() if args.graph else None
    trace = None
    if args.trace:
        ctas = m.step_kernel_ctas()
        trace = torch.zeros((ctas, args.trace_cap, 4), dtype=torch.int64, device="cuda")
        m.set_step_trace(trace)
    times = []
    for k in range(args.steps):
        if trace is not None:
            trace.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if st is not None:
            a.record(st)
            m.decoder_step(ids, stream=st)
            b.record(st)
        else:
            a.record()
            m.decoder_step(ids)
            b.record()
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b))
    assert m.poll_device_error() == 0
    if trace is not None:
        rec = trace.cpu().numpy()
        np.save(args.trace, rec)
        print(json.dumps(trace_summary(rec, cfg.n_dec)))
    ts = [np.full(B, args.t + k) for k in range(args.steps)]
    byts = [roofline.decoder_step_bytes(cfg, x) for x in ts]
    print(json.dumps({"workload": args.workload, "batch": B, "t": args.t, "graph": args.graph,
                      "kernel": "fused" if m.get_step_kernel() == 1 else "chain",
                      "step_kernel_ctas": m.step_kernel_ctas(),
                      "step_ms": times, "step_GB": [x / 1e9 for x in byts],
                      "GB_s": [x / (ms / 1e3) / 1e9 for x, ms in zip(byts, times)]}))


PHASES = {0: "qkv", 0x81: "swa", 2: "wo", 3: "wqx", 0x84: "xattn", 5: "wox", 6: "ffn1",
          7: "ffn1b", 8: "ffn2"}


def trace_summary(rec, n_dec):
    """Where a persistent step's time goes, from its trace records
    [ctas][cap][4] = (item id, start, dependency met, end): per item kind,
    the mean over layers and row tiles of the span from the first CTA's
    start to the last CTA's end, of the part after the last dependency was
    met, and of the CTA-busy time per item."""
    r = rec.reshape(-1, 4)
    r = r[r[:, 0] != 0]
    if not len(r):
        return {"trace": "empty"}
    t0 = r[:, 1].min()
    groups = {}
    for idv, a, dp, e in r:
        groups.setdefault(int(idv), []).append((a - t0, dp - t0, e - t0))
    kinds = {}
    for idv, items in groups.items():
        layer, ph, row = (idv >> 16) - 1, (idv >> 8) & 0xFF, idv & 0xFF
        name = PHASES.get(ph, "pre" if layer == n_dec else str(ph))
        if layer == n_dec:
            name = {1: "gate", 0x20: "gather", 0x21: "final"}.get(ph, name)
        x = np.asarray(items, dtype=np.float64)
        k = kinds.setdefault(name, {"span": [], "after_dep": [], "busy": [], "items": 0})
        k["span"].append(x[:, 2].max() - x[:, 0].min())
        k["after_dep"].append(x[:, 2].max() - x[:, 1].max())
        k["busy"].append(float(np.mean(x[:, 2] - x[:, 1])))
        k["items"] += len(items)
    out = {name: {"groups": len(v["span"]), "items": v["items"],
                  "span_us": round(float(np.mean(v["span"])) / 1e3, 2),
                  "after_last_dep_us": round(float(np.mean(v["after_dep"])) / 1e3, 2),
                  "busy_per_item_us": round(float(np.mean(v["busy"])) / 1e3, 2)}
           for name, v in kinds.items()}
    out["kernel_us"] = round(float(r[:, 3].max() - t0) / 1e3, 1)
    return out


def run_attend(args):
    import torch

    from . import rlt
    n, H, dh, cap = args.n, args.heads, args.dh, args.cap
    L = args.len or cap
    g = torch.Generator(device="cuda").manual_seed(3)
    q = torch.randn((n, H, dh), generator=g, device="cuda")
    kv = torch.randn((n, H, 2, cap, dh), generator=g, device="cuda").to(torch.bfloat16)
    out = torch.empty((n, H, dh), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(rlt.attend_workspace_bytes(n, H, dh, cap), dtype=torch.uint8,
                     device="cuda")
    lengths = [L] * n
    times = []
    for _ in range(args.reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        rlt.attend(q, kv, lengths, out, ws)
        b.record()
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b))
    byts = n * H * 2 * L * dh * 2
    print(json.dumps({"attend": [n, H, dh, cap, L], "ms": times, "GB": byts / 1e9,
                      "GB_s": [byts / (t / 1e3) / 1e9 for t in times]}))


def run_parallel(args):
    """Encoder prefill, then the token-parallel decoder pass (feedback-off
    workloads), `--steps` times; prints each pass's CUDA-event time."""
    import torch

    from . import configs, inputs
    from .rlt import Model
    wl = configs.workloads()[args.workload]
    cfg = wl.model
    B = args.batch or wl.batch
    T = args.max_len or wl.max_len
    lengths = [T] * B
    w = inputs.make_weights(cfg)
    tok = inputs.make_tokens(cfg.vocab, lengths)
    m = Model(cfg, w, B, T)
    del w
    flat = torch.from_numpy(tok.reshape(-1).astype(np.int32)).cuda()
    offsets = np.arange(B, dtype=np.int32) * T
    ids = list(range(B))
    times = []
    for _ in range(args.steps):
        m.prefill_encoder(flat, ids, offsets, lengths)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        m.decoder_parallel(ids, T)
        b.record()
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b))
    assert m.poll_device_error() == 0
    print(json.dumps({"workload": args.workload, "batch": B, "T": T, "parallel_ms": times}))


def run_backward(args):
    """Backpropagation through time over the first `--max-len` positions of
    the batch (rlt_backward: recorded forward, reverse traversal, memory
    gradient), `--steps` times from the same start state; prints each call's
    CUDA-event time and seq-steps/s."""
    import torch

    from . import configs, inputs, roofline
    from .rlt import Model
    wl = configs.workloads()[args.workload]
    cfg = wl.model
    if args.layers:
        cfg = cfg.replace(n_enc=args.layers, n_dec=args.layers,
                          mem_groups=1 if cfg.mem_groups == 1 else args.layers)
    B = args.batch or wl.batch
    T = args.max_len or wl.max_len
    lengths = [T] * B
    w = inputs.make_weights(cfg)
    tok = inputs.make_tokens(cfg.vocab, lengths)
    m = Model(cfg, w, B, T)
    del w
    flat = torch.from_numpy(tok.reshape(-1).astype(np.int32)).cuda()
    ids = list(range(B))
    m.prefill_encoder(flat, ids, np.arange(B, dtype=np.int32) * T, lengths)
    t0 = args.bw_start  # the chunk covers positions t0 .. T-1
    if t0:
        m.run_sequence(ids, t0)
    start = [m.get_state(i) for i in ids]
    NS = T - t0
    sgrad = torch.randn((B, NS, cfg.d), device="cuda", generator=torch.Generator("cuda").manual_seed(3))
    ws = torch.empty(m.backward_workspace_bytes(B, NS), dtype=torch.uint8, device="cuda")
    grads = {k: torch.zeros(v, device="cuda") for k, v in m.grad_shapes().items()}
    egrad = torch.zeros((B, T, cfg.d), device="cuda")
    times = []
    for _ in range(args.steps):
        for i, (s, c, t) in zip(ids, start):
            m.set_state(i, s, c, t)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        m.backward(ids, sgrad, grads=grads, egrad=egrad, workspace=ws)
        b.record()
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b))
    assert m.poll_device_error() == 0
    flops = roofline.backward_flops(cfg, lengths)
    best = min(times)
    print(json.dumps({"workload": args.workload, "batch": B, "T": T, "start": t0,
                      "backward_ms": times, "seq_steps_per_s": B * NS / (best / 1e3),
                      "tflops": flops / (best / 1e3) / 1e12,
                      "workspace_gb": ws.numel() / 1e9}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="m140_bf16")
    ap.add_argument("--t", type=int, default=512)
    ap.add_argument("--steps", type=int, default=2)
    ap.add_argument("--batch", type=int, default=0)
    ap.add_argument("--max-len", type=int, default=0,
                    help="sequence length of the arena (default: the workload's); small "
                         "values keep a profiler's device memory small")
    ap.add_argument("--graph", action="store_true")
    ap.add_argument("--layers", type=int, default=0,
                    help="encoder and decoder blocks (default: the workload's)")
    ap.add_argument("--trace", default="",
                    help="record the persistent step's work items into this .npy file and "
                         "print where the time goes (last step)")
    ap.add_argument("--trace-cap", type=int, default=1024)
    ap.add_argument("--kernel", choices=["fused", "chain"], default=None,
                    help="decoder step kernel (default: the model's default)")
    ap.add_argument("--attend", action="store_true")
    ap.add_argument("--backward", action="store_true",
                    help="time rlt_backward over --max-len positions of --batch sequences")
    ap.add_argument("--bw-start", type=int, default=0,
                    help="backward chunk starts at this position (the forward runs there first)")
    ap.add_argument("--parallel", action="store_true",
                    help="time the token-parallel decoder pass (feedback-off workloads)")
    ap.add_argument("--n", type=int, default=256)
    ap.add_argument("--heads", type=int, default=12)
    ap.add_argument("--dh", type=int, default=64)
    ap.add_argument("--cap", type=int, default=1024)
    ap.add_argument("--len", type=int, default=0)
    ap.add_argument("--reps", type=int, default=3)
    args = ap.parse_args()
    if args.attend:
        run_attend(args)
    elif args.parallel:
        run_parallel(args)
    elif args.backward:
        run_backward(args)
    else:
        run_steps(args)


if __name__ == "__main__":
    main()
