#!/usr/bin/env python3
"""Benchmark: predictor-gated sparse FFN, tokens/s per layer stack at batch 1.

Workload (default): the OPT-6.7B-shaped ReLU FFN stack -- 32 layers,
d_model 4096, d_ff 16384, predictor rank 1024, fp16 weights, Zipf(1.1)
firing profile at 20% mean activation -- run on its 128 synthetic decode
tokens at batch 1, one token after the other.  One step = those 128 tokens
through all 32 layers (predict -> compact -> gathered FFN -> residual), replayed
from a CUDA graph.  The weights (9.5 GB) are far larger than the 126 MB L2, so
every step streams them from HBM.

Also reported on the same GPU:
  roofline     the gathered-FFN kernel: algorithmic bytes / kernel time, with
               CUDA events recorded around every launch inside the timed graph
  dense        the same FFN with every neuron (no predictor): the speedup
               denominator
  mode_F       the predictor calibrated to the true firing fraction
  e2e          the public API called eagerly per token, with the step's
               tokens copied from pinned host memory and results copied back
  cpu_baseline the fp64 oracle on the host cores (bounded sample)

`--impl reference` times the fp64 oracle on the host cores instead.
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "sparse-FFN tokens/s per layer stack at batch 1; achieved HBM GB/s vs roofline"
UNIT = "tokens/s"
FALLBACK_HBM_GBS = 6650.0

# DRAM traffic of one gathered-FFN launch from an ncu capture, as a ratio to the
# launch's algorithmic bytes, with the hash of the kernel sources it was taken
# on (a changed kernel invalidates it).
TRAFFIC = {"ratio": 1.187, "src_sha": "0ab03e39e107de07",
           "profile": "profiles/k_ffn_ldg_k_predict_opt67b_2layer.md"}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="opt-6.7b")
    ap.add_argument("--mode", default="R", choices=["R", "F"])
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--layers", type=int, default=0,
                    help="use only the first N layers of the stack (a small case for profiling)")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip dense, mode F, e2e and CPU baseline legs")
    ap.add_argument("--cpu-seconds", type=float, default=20.0)
    ap.add_argument("--counts-out", default="",
                    help="write the active-neuron count and algorithmic bytes of every "
                         "gathered-FFN launch of one step (token x layer) as JSON")
    return ap.parse_args()


def env_rank():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def max_over_ranks(ms, world, device):
    """The slowest rank's time: a step ends when every replica has finished."""
    if world <= 1:
        return ms
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_value(tokens_per_rank, world, ms):
    """Whole-job throughput: the tokens of all replicas over the slowest time."""
    return world * tokens_per_rank / (ms / 1e3)


def src_sha():
    h = hashlib.sha256()
    d = os.path.join(ROOT, "activation_sparse_pi_b200", "csrc")
    for f in sorted(os.listdir(d)):
        h.update(open(os.path.join(d, f), "rb").read())
    return h.hexdigest()[:16]


def measured_hbm():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def workload_config(cfg, mode, B):
    return {
        "workload": (f"{cfg.name}-shaped {cfg.act} FFN stack: {cfg.n_layers} layers, d_model "
                     f"{cfg.d_model}, d_ff {cfg.d_ff}, predictor rank {cfg.rank}, {cfg.wdtype} "
                     f"weights, batch {B}, {cfg.n_tokens} decode tokens per step"),
        "predictor_mode": mode,
        "batch": B,
        "tokens_per_step": cfg.n_tokens,
        "layers": cfg.n_layers,
        "l2": "inputs larger than L2: every step streams the stack's weights from HBM",
        "parallelism": "replicas (one independent stack per GPU)",
    }


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during a region."""

    Q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, dev_id):
        self.dev_id = dev_id
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.dev_id, f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 7:
                continue
            try:
                sm.append(float(f[0]))
                mx = float(f[1])
            except ValueError:
                continue
            for n, v in zip(names, f[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ helpers
def host_oracle_layer(L):
    """LayerData (any device) -> oracle.OracleLayer with host copies."""
    import numpy as np
    import torch

    import oracle

    def raw(t):
        if t is None:
            return None
        t = t.detach().cpu()
        if t.dtype in (torch.float16, torch.bfloat16):
            return t.contiguous().view(torch.int16).numpy().view(np.uint16)
        if t.dtype == torch.uint8:
            return t.numpy()
        return t.double().numpy()

    c = L.cfg
    return oracle.OracleLayer(
        d_model=c.d_model, d_ff=c.d_ff, act=c.act, wdtype=c.wdtype, pdtype=c.adtype,
        w1=raw(L.w1), b1=raw(L.b1), w2=raw(L.w2), b2=raw(L.b2), threshold=float(L.threshold),
        w_up=raw(L.w_up), w_gate=raw(L.w_gate), w_down_t=raw(L.w_down_t), b_up=raw(L.b_up),
        b_gate=raw(L.b_gate))


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def oracle_sample(layers_host_fn, cfg, budget_s, token):
    """Time the oracle's stack on one token, layer by layer, until the budget
    is spent.  Returns (tokens/s per stack, layers timed, seconds)."""
    import numpy as np

    import oracle

    x = np.asarray(token, dtype=np.float64).reshape(1, -1)
    spent, done = 0.0, 0
    for l in range(cfg.n_layers):
        OL = layers_host_fn(l)
        t0 = time.perf_counter()
        xl = oracle.rms_cast(x, cfg.adtype)
        y, _, _ = oracle.sparse_ffn_layer(OL, xl)
        x = x + y
        spent += time.perf_counter() - t0
        done += 1
        if spent >= budget_s:
            break
    per_layer = spent / done
    return 1.0 / (per_layer * cfg.n_layers), done, spent


def layer_bytes(cfg):
    """(row bytes of one FFN matrix, matrices per neuron)."""
    rb = cfg.d_model // 32 * 18 if cfg.wdtype == "q4_0" else cfg.d_model * 2
    return rb, (3 if cfg.act == "reglu" else 2)


def ffn_launch_bytes(cfg, K, B):
    """Algorithmic bytes of one gathered-FFN launch over K neurons: every
    gathered row once, the neuron's bias and index, the input activations and
    the output."""
    rb, nm = layer_bytes(cfg)
    return K * (nm * rb + 4 + 4) + B * cfg.d_model * 2 + B * cfg.d_model * 4


def predictor_bytes(cfg):
    return cfg.rank * cfg.d_model * 2 + cfg.rank * 4 + cfg.d_ff * cfg.rank * 2 + cfg.d_ff * 4


# ------------------------------------------------------------------ our arm
def run_ours(args, rank, world, local):
    import numpy as np
    import torch

    import activation_sparse_pi_b200 as pi
    import synth
    from activation_sparse_pi_b200 import build as pibuild

    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group(
            "nccl", timeout=datetime.timedelta(seconds=300), device_id=torch.device("cuda", local))
    pibuild.build()
    pi.lib()
    cfg = synth.get_config(args.config)
    if args.layers:
        import dataclasses
        cfg = dataclasses.replace(cfg, n_layers=min(args.layers, cfg.n_layers))
    B, T, NL, d, F = args.batch, cfg.n_tokens, cfg.n_layers, cfg.d_model, cfg.d_ff

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    # ---- workload, generated on this GPU
    layers = [synth.make_layer(cfg, l, "cuda", args.mode) for l in range(NL)]

    def descs_for(ls):
        ds = [pi.layer_from_tensors(
            d_model=d, d_ff=F, rank=cfg.rank, wdtype=cfg.wdtype, adtype=cfg.adtype, act=cfg.act,
            w1=L.w1, b1=L.b1, w2=L.w2, b2=L.b2, threshold=L.threshold, w_up=L.w_up,
            w_gate=L.w_gate, w_down_t=L.w_down_t, b_up=L.b_up, b_gate=L.b_gate) for L in ls]
        return pi.layer_array(ds)

    arr = descs_for(layers)
    ws = torch.empty(pi.pi_workspace_size(arr, B), dtype=torch.uint8, device="cuda")
    X0 = synth.make_tokens(cfg, T * B).reshape(T, B, d).cuda()
    Xw = torch.empty_like(X0)

    def step_graph(arr_, timed_events=None, counts=None):
        # eager call first: kernel attributes are set outside the capture
        Xw.copy_(X0)
        pi.pi_ffn_stack(arr_, Xw[0], B, None, None, ws)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        n0 = pi.pi_launch_count()
        with torch.cuda.graph(g):
            Xw.copy_(X0)
            for t in range(T):
                if timed_events is None:
                    pi.pi_ffn_stack(arr_, Xw[t], B, None, None, ws)
                else:
                    pi.pi_ffn_stack_timed(arr_, Xw[t], B, None, counts[t], ws, timed_events[t])
        return g, pi.pi_launch_count() - n0

    def time_graph(g, steps, warmup):
        for _ in range(warmup):
            g.replay()
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(steps):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        barrier()
        return max_over_ranks(e0.elapsed_time(e1), world, "cuda")

    # ---- headline: graph replay of the step
    g, launches_per_step = step_graph(arr)
    dev_id = "GPU-" + str(torch.cuda.get_device_properties(local).uuid)
    for _ in range(args.warmup):
        g.replay()
    torch.cuda.synchronize()
    with ClockSampler(dev_id) as clk:
        ms = time_graph(g, args.steps, 0)
    clocks = clk.summary()
    assert pi.pi_device_error() == 0, "device-side error flagged during the timed region"
    value = job_value(args.steps * T * B, world, ms)
    out_sample = Xw.float().cpu()
    assert torch.isfinite(out_sample).all()
    del g

    # ---- roofline of the gathered-FFN kernel: events around every launch
    counts = torch.zeros(T, NL, dtype=torch.int32, device="cuda")
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * NL)] for _ in range(T)]
    for row in evs:  # torch creates the CUDA event on first record
        for e in row:
            e.record()
    torch.cuda.synchronize()
    gt, _ = step_graph(arr, evs, counts)
    gt.replay()
    torch.cuda.synchronize()
    tstart = torch.cuda.Event(enable_timing=True)
    tend = torch.cuda.Event(enable_timing=True)
    tstart.record()
    gt.replay()
    tend.record()
    torch.cuda.synchronize()
    timed_step_ms = tstart.elapsed_time(tend)
    durs = np.array([[evs[t][2 * l].elapsed_time(evs[t][2 * l + 1]) for l in range(NL)]
                     for t in range(T)])
    Ks = counts.cpu().numpy().astype(np.int64)
    ffn_bytes = np.vectorize(lambda k: ffn_launch_bytes(cfg, int(k), B))(Ks)
    achieved = float(ffn_bytes.sum() / (durs.sum() / 1e3)) / 1e9
    peak, peak_kind = measured_hbm()
    ffn_bytes_per_launch = float(ffn_bytes.mean())
    traffic = None
    if TRAFFIC and TRAFFIC.get("src_sha") == src_sha():
        traffic = round(TRAFFIC["ratio"] * ffn_bytes_per_launch)
    roofline = {
        "bound": "hbm", "kernel": "k_ffn (gathered up + down)", "achieved": round(achieved, 1),
        "peak": peak, "unit": "GB/s", "frac": round(achieved / peak, 4),
        "peak_kind": peak_kind,
        "traffic": traffic, "algorithmic_bytes_per_launch": round(ffn_bytes_per_launch),
        "avg_launch_us": round(float(durs.mean()) * 1e3, 2),
        "launches_timed": int(durs.size),
        "mean_active_frac": round(float(Ks.mean()) / F, 4),
    }
    # whole-stack algorithmic bytes per step (predictor + gathered rows + activations)
    stack_bytes = float(ffn_bytes.sum()) + T * NL * (predictor_bytes(cfg) + B * d * 4 * 2)
    stack_gbs = stack_bytes / (ms / args.steps / 1e3) / 1e9
    stack = {"achieved": round(stack_gbs, 1), "unit": "GB/s", "peak": peak,
             "frac": round(stack_gbs / peak, 4), "bytes_per_step": round(stack_bytes),
             "timed_graph_step_ms": round(timed_step_ms, 3)}
    del gt, evs
    if args.counts_out and rank == 0:
        with open(args.counts_out, "w") as f:
            json.dump({"order": "token-major, then layer", "counts": Ks.tolist(),
                       "algorithmic_bytes": ffn_bytes.tolist(),
                       "event_us": (durs * 1e3).round(3).tolist()}, f)

    extras = {}
    if not args.no_extras:
        # ---- dense denominator: every neuron, no predictor, same FFN kernels
        idx_all = torch.arange(F, dtype=torch.int32, device="cuda")
        cnt_all = torch.tensor([F], dtype=torch.int32, device="cuda")
        x16 = torch.randn(B, d, device="cuda").to(torch.bfloat16 if cfg.adtype == "bf16"
                                                   else torch.float16)
        y = torch.empty(B, d, dtype=torch.float32, device="cuda")
        for l in range(NL):
            pi.pi_sparse_ffn(arr[l], x16, B, idx_all, cnt_all, y, ws)
        torch.cuda.synchronize()
        gd = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gd):
            for t in range(T):
                for l in range(NL):
                    pi.pi_sparse_ffn(arr[l], x16, B, idx_all, cnt_all, y, ws)
        dreps = 3
        dms = time_graph(gd, dreps, 1)
        dense_tps = job_value(dreps * T * B, world, dms)
        extras["dense"] = {"value": round(dense_tps, 2), "unit": UNIT,
                           "speedup_sparse_over_dense": round(value / dense_tps, 3)}
        del gd

        # ---- mode F: same weights, predictor calibrated to the firing fraction
        other = "F" if args.mode == "R" else "R"
        layers_o = [synth.with_mode(L, other) for L in layers]
        arr_o = descs_for(layers_o)
        go, _ = step_graph(arr_o)
        oms = time_graph(go, max(3, args.steps // 2), 1)
        cnt_o = torch.zeros(NL, dtype=torch.int32, device="cuda")
        Xw.copy_(X0)
        pi.pi_ffn_stack(arr_o, Xw[0], B, None, cnt_o, ws)
        extras["mode_" + other] = {
            "value": round(job_value(max(3, args.steps // 2) * T * B, world, oms), 2),
            "unit": UNIT, "mean_active_frac_token0": round(float(cnt_o.float().mean()) / F, 4)}
        del go, layers_o, arr_o

        # ---- e2e: public API, eager, host buffers in and out every step
        Xh = X0.cpu().pin_memory()
        Oh = torch.empty_like(Xh).pin_memory()

        def e2e_step():
            Xw.copy_(Xh, non_blocking=True)
            for t in range(T):
                pi.pi_ffn_stack(arr, Xw[t], B, None, None, ws)
            Oh.copy_(Xw, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        esteps = max(3, args.steps // 4)
        e0.record()
        for _ in range(esteps):
            e2e_step()
        e1.record()
        torch.cuda.synchronize()
        ems = max_over_ranks(e0.elapsed_time(e1), world, "cuda")
        nbytes = Xh.numel() * Xh.element_size()
        extras["e2e"] = {"value": round(job_value(esteps * T * B, world, ems), 2), "unit": UNIT,
                         "h2d_bytes_per_step": nbytes, "d2h_bytes_per_step": nbytes,
                         "steps": esteps, "api": "pi_ffn_stack per token, eager launches"}

        # ---- oracle on the host cores (rank 0 of a 1-GPU run)
        if rank == 0 and world == 1:
            tps, nl_done, secs = oracle_sample(lambda l: host_oracle_layer(layers[l]), cfg,
                                               args.cpu_seconds, X0[0].cpu().numpy())
            extras["cpu_baseline"] = {
                "value": round(tps, 5), "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                "sample": (f"one token through the first {nl_done} of {NL} layers in fp64 "
                           f"({secs:.1f} s), scaled to the whole stack")}

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": cfg.wdtype,
            "data": "synthetic", "config": workload_config(cfg, args.mode, B),
            "roofline": roofline, "stack_roofline": stack,
            "gpu_launches": int(launches_per_step * args.steps),
            "clocks": clocks,
        }
        for k in ("cpu_baseline", "e2e"):
            if k in extras:
                line[k] = extras.pop(k)
        line.update(extras)
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


# ------------------------------------------------------------- reference arm
def run_reference(args, rank, world, local):
    """The fp64 oracle on the host cores; each step is one layer of the stack
    for one token (a bounded sample), carrying the residual stream."""
    if rank != 0:
        return
    import numpy as np
    import torch

    import oracle
    import synth

    cfg = synth.get_config(args.config)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    if dev == "cuda":
        torch.cuda.set_device(local)
    nl = min(cfg.n_layers, args.steps + args.warmup)
    cache = {}

    def host_layer(l):
        if l not in cache:
            cache[l] = host_oracle_layer(synth.make_layer(cfg, l, dev, args.mode))
            if dev == "cuda":
                torch.cuda.empty_cache()
        return cache[l]

    for l in range(nl):
        host_layer(l)
    x = synth.make_tokens(cfg, args.batch).double().numpy()
    times = []
    for s in range(args.warmup + args.steps):
        l = s % nl
        t0 = time.perf_counter()
        xl = oracle.rms_cast(x, cfg.adtype)
        y, _, _ = oracle.sparse_ffn_layer(host_layer(l), xl)
        x = x + y
        dt = time.perf_counter() - t0
        if s >= args.warmup:
            times.append(dt)
    per_layer = float(np.mean(times))
    value = args.batch / (per_layer * cfg.n_layers)
    sample = (f"each step: one layer (cycling over the first {nl} of {cfg.n_layers}) for "
              f"{args.batch} token(s) in fp64; tokens/s scaled to the {cfg.n_layers}-layer stack")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 5), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(per_layer * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(cfg, args.mode, args.batch),
        "cpu_baseline": {"value": round(value, 5), "unit": UNIT, "cores": blas_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 5), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    rank, world, local = env_rank()
    if args.impl == "reference":
        run_reference(args, rank, world, local)
    else:
        run_ours(args, rank, world, local)


if __name__ == "__main__":
    main()
