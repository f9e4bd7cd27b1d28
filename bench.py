#!/usr/bin/env python3
"""Benchmark: predictor-gated sparse FFN, tokens/s per layer stack at batch 1.

Headline workload (default): the Falcon(ReLU)-40B-shaped FFN stack, the
largest configuration that fits one GPU -- 60 layers, d_model 8192, d_ff
32768, predictor rank 1024, fp16 weights (64.4 GB of FFN weights plus 5 GB of
predictors, all resident in HBM), Zipf(1.0) firing profile at 8% mean
activation, predictor calibrated to recall 0.9 -- run on its 128 synthetic
decode tokens at batch 1, one token after the other.  One step = those 128
tokens through all 60 layers (predict -> compact -> gathered FFN ->
residual), replayed from a CUDA graph.  The weights are far larger than the
126 MB L2, so every step streams them from HBM.

Also reported on the same GPU:
  roofline       the gathered-FFN kernel: algorithmic bytes / kernel time,
                 CUDA events recorded around every launch inside the timed graph
  stack_roofline the whole step: predictor + active-row + activation bytes
  dense          the same FFN with every neuron (no predictor): the speedup
                 denominator
  mode_F         the predictor calibrated to the true firing fraction
  prompt_b64     the 64-token prompt as one batch-64 union step
  e2e            the public API called eagerly per token, with the step's
                 tokens copied from pinned host memory and results copied back
  parity_sample  token 0 through the first layers, each layer checked against
                 the fp64 oracle fed the GPU's own residual (band neurons
                 counted)
  cpu_baseline   the single-threaded fp64 C++ oracle on the host (same sample)
  configs        the other workloads (OPT-6.7B, its Squared-ReLU variant,
                 ReLU-Llama-2-13B at batch 1 and 8, LLaMA-70B Q4_0 at batch 1,
                 8 and 32), each on the first layers of its stack

`--impl reference` times the fp64 oracle on the host cores instead.
"""
import argparse
import dataclasses
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
NOMINAL_HBM_GBS = 8000.0  # the ~8 TB/s HBM3e figure the roofline target is quoted against
SAMPLE_LAYERS = 4         # layers of the oracle sample (both arms)

# DRAM traffic of one gathered-FFN launch from an ncu capture, as a ratio to the
# launch's algorithmic bytes, with the hash of the sources that define the
# kernel (k_ffn_ldg: pi_common.cuh, pi_predict.cuh, pi_ffn.cuh) when it was
# taken; a changed kernel invalidates it.
TRAFFIC = {"ratio": 1.074, "src_sha": "f8e9a7df2cab9f58", "config": "falcon-40b",
           "files": ("pi_common.cuh", "pi_predict.cuh", "pi_ffn.cuh"),
           "profile": "profiles/k_ffn_ldg_falcon40b_2layer.md"}

# other workloads: (key, config, batch, layers of the stack timed)
EXTRAS = [
    ("opt-6.7b_b1", "opt-6.7b", 1, 32),
    ("opt-6.7b-sqrelu_b1", "opt-6.7b-sqrelu", 1, 8),
    ("opt-6.7b-adaptive_b1", "opt-6.7b-adaptive", 1, 32),
    ("relu-llama2-13b_b1", "relu-llama2-13b", 1, 10),
    ("relu-llama2-13b_b8", "relu-llama2-13b", 8, 10),
    ("llama2-70b-q4_b1", "llama2-70b-q4", 1, 10),
    ("llama2-70b-q4_b8", "llama2-70b-q4", 8, 10),
    ("llama2-70b-q4_b32", "llama2-70b-q4", 32, 10),
]


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="falcon-40b")
    ap.add_argument("--mode", default="R", choices=["R", "F"])
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--layers", type=int, default=0,
                    help="use only the first N layers of the stack (a small case for profiling)")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the dense, mode F, prompt, e2e, oracle and other-config legs")
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


def src_sha(files):
    h = hashlib.sha256()
    d = os.path.join(ROOT, "activation_sparse_pi_b200", "csrc")
    for f in files:
        h.update(open(os.path.join(d, f), "rb").read())
    return h.hexdigest()[:16]


def measured_hbm():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def host_info():
    model = ""
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    model = ln.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    try:
        nproc = len(os.sched_getaffinity(0))
    except AttributeError:
        nproc = os.cpu_count() or 1
    return {"nproc": nproc, "cpu_model": model}


def workload_config(cfg, mode, B, n_layers=None, tokens=None):
    L = n_layers or cfg.n_layers
    T = tokens or cfg.n_tokens
    return {
        "workload": (f"{cfg.name}-shaped {cfg.act} FFN stack: {L} layers, d_model "
                     f"{cfg.d_model}, d_ff {cfg.d_ff}, predictor rank {cfg.rank}, {cfg.wdtype} "
                     f"weights, batch {B}, {T} decode tokens per step"),
        "predictor_mode": mode,
        "batch": B,
        "tokens_per_step": T,
        "layers": L,
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


def predictor_bytes(cfg, rank=None):
    r = cfg.rank if rank is None else rank
    return r * cfg.d_model * 2 + r * 4 + cfg.d_ff * r * 2 + cfg.d_ff * 4


# ------------------------------------------------------------------ our arm
class Stack:
    """One generated layer stack on this GPU, with its descriptors and a
    workspace, and the means to time a step over it."""

    def __init__(self, cfg, mode, B, world):
        import torch

        import activation_sparse_pi_b200 as pi
        import synth
        self.torch, self.pi, self.synth = torch, pi, synth
        self.cfg, self.mode, self.B, self.world = cfg, mode, B, world
        self.layers = [synth.make_layer(cfg, l, "cuda", mode) for l in range(cfg.n_layers)]
        self.arr = self.descs(self.layers)
        self.ws = torch.empty(pi.pi_workspace_size(self.arr, B), dtype=torch.uint8,
                              device="cuda")

    def with_batch(self, B):
        """The same layers and descriptors, run at another batch size."""
        other = Stack.__new__(Stack)
        other.__dict__.update(self.__dict__)
        other.B = B
        other.ws = self.torch.empty(self.pi.pi_workspace_size(self.arr, B),
                                    dtype=self.torch.uint8, device="cuda")
        return other

    def hot_first(self):
        """The same stack with every layer's neurons renumbered hottest first
        (pi_permute_layer), ordered by the generator's firing profile -- what
        an offline activation profiler would measure."""
        import numpy as np
        torch, pi, synth = self.torch, self.pi, self.synth
        other = Stack.__new__(Stack)
        other.__dict__.update(self.__dict__)
        keys = ("w_up", "w_gate", "w_down_t", "w2", "b2", "b_up", "b_gate")
        layers = []
        for l, L in enumerate(self.layers):
            kw = dict(L.__dict__)
            for k in keys:
                v = getattr(L, k)
                kw[k] = None if v is None else torch.empty_like(v)
            P = synth.LayerData(**kw)
            perm = torch.from_numpy(np.argsort(-L.p, kind="stable").astype(np.int32)).cuda()
            pi.pi_permute_layer(self.arr[l], perm, self.descs([P])[0])
            layers.append(P)
        torch.cuda.synchronize()
        other.layers = layers
        other.arr = other.descs(layers)
        return other

    def descs(self, ls):
        c = self.cfg
        return self.pi.layer_array([self.pi.layer_from_tensors(
            d_model=c.d_model, d_ff=c.d_ff, rank=L.w1.shape[0], wdtype=c.wdtype, adtype=c.adtype,
            act=c.act, w1=L.w1, b1=L.b1, w2=L.w2, b2=L.b2, threshold=L.threshold, w_up=L.w_up,
            w_gate=L.w_gate, w_down_t=L.w_down_t, b_up=L.b_up, b_gate=L.b_gate) for L in ls])

    def tokens(self, T, seed_offset=0):
        """T synthetic tokens as [T/B, B, d] fp32 on the device."""
        c = self.cfg
        return self.synth.make_tokens(c, T, seed_offset=seed_offset).reshape(
            T // self.B, self.B, c.d_model).cuda()

    def graph(self, arr, X0, Xw, timed_events=None, counts=None):
        torch, pi = self.torch, self.pi
        Xw.copy_(X0)
        pi.pi_ffn_stack(arr, Xw[0], self.B, None, None, self.ws)  # kernel attributes set eagerly
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        n0 = pi.pi_launch_count()
        with torch.cuda.graph(g):
            Xw.copy_(X0)
            for t in range(X0.shape[0]):
                if timed_events is None:
                    pi.pi_ffn_stack(arr, Xw[t], self.B, None, None, self.ws)
                else:
                    pi.pi_ffn_stack_timed(arr, Xw[t], self.B, None, counts[t], self.ws,
                                          timed_events[t])
        return g, pi.pi_launch_count() - n0

    def time_graph(self, g, steps, warmup, barrier=None):
        torch = self.torch
        for _ in range(warmup):
            g.replay()
        torch.cuda.synchronize()
        if barrier:
            barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(steps):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        if barrier:
            barrier()
        return max_over_ranks(e0.elapsed_time(e1), self.world, "cuda")

    def ffn_roofline(self, X0, Xw, peak):
        """CUDA events around every gathered-FFN launch of one graph replay."""
        import numpy as np
        torch, cfg = self.torch, self.cfg
        NT, NL = X0.shape[0], cfg.n_layers
        counts = torch.zeros(NT, NL, dtype=torch.int32, device="cuda")
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * NL)] for _ in range(NT)]
        for row in evs:  # torch creates the CUDA event on first record
            for e in row:
                e.record()
        torch.cuda.synchronize()
        gt, _ = self.graph(self.arr, X0, Xw, evs, counts)
        gt.replay()
        torch.cuda.synchronize()
        gt.replay()
        torch.cuda.synchronize()
        durs = np.array([[evs[t][2 * l].elapsed_time(evs[t][2 * l + 1]) for l in range(NL)]
                         for t in range(NT)])
        Ks = counts.cpu().numpy().astype(np.int64)
        fb = np.vectorize(lambda k: ffn_launch_bytes(cfg, int(k), self.B))(Ks)
        achieved = float(fb.sum() / (durs.sum() / 1e3)) / 1e9
        del gt, evs
        return {
            "bound": "hbm", "kernel": "gathered FFN (up + down, one launch at batch 1-4)",
            "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4),
            "frac_of_nominal_8tbs": round(achieved / NOMINAL_HBM_GBS, 4),
            "algorithmic_bytes_per_launch": round(float(fb.mean())),
            "avg_launch_us": round(float(durs.mean()) * 1e3, 2),
            "launches_timed": int(durs.size),
            "mean_active_frac": round(float(Ks.mean()) / cfg.d_ff, 4),
        }, Ks, fb, durs

    def step_bytes(self, fb_sum, n_batches):
        """Algorithmic bytes of one step: gathered rows and activations (fb_sum)
        plus every layer's predictor and the residual read and written."""
        c = self.cfg
        per_token = sum(predictor_bytes(c, L.w1.shape[0]) for L in self.layers)
        return float(fb_sum) + n_batches * (per_token + c.n_layers * self.B * c.d_model * 4 * 2)


def measure(stack, T, steps, warmup, peak, barrier=None, seed_offset=0):
    """tokens/s of a step over T tokens, the FFN roofline and the stack roofline."""
    torch = stack.torch
    X0 = stack.tokens(T, seed_offset)
    Xw = torch.empty_like(X0)
    g, launches = stack.graph(stack.arr, X0, Xw)
    ms = stack.time_graph(g, steps, warmup, barrier)
    del g
    roof, Ks, fb, durs = stack.ffn_roofline(X0, Xw, peak)
    step_s = ms / steps / 1e3
    sb = stack.step_bytes(fb.sum(), X0.shape[0])
    return {
        "value": round(job_value(steps * T, stack.world, ms), 2), "unit": UNIT,
        "ms_per_step": round(ms / steps, 4), "tokens_per_step": T,
        "roofline": roof,
        "stack_roofline": {"achieved": round(sb / step_s / 1e9, 1), "unit": "GB/s",
                           "peak": peak, "frac": round(sb / step_s / 1e9 / peak, 4),
                           "frac_of_nominal_8tbs": round(sb / step_s / 1e9 / NOMINAL_HBM_GBS, 4),
                           "bytes_per_step": round(sb)},
    }, launches, (Ks, fb, durs)


def parity_and_cpu_sample(stack, x_tok, n_layers, budget_s):
    """Token 0 through the first layers of the stack on the GPU, one layer at a
    time, and each layer through the fp64 oracle fed the GPU's own residual
    (teacher forcing).  Returns (parity summary, oracle seconds per layer,
    layers timed).  Only the oracle's layer computation is timed."""
    import numpy as np
    import torch

    import oracle
    pi, cfg = stack.pi, stack.cfg
    F = cfg.d_ff
    xr = x_tok.reshape(1, -1).clone().cuda()
    idx = torch.zeros(1, F, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(1, dtype=torch.int32, device="cuda")
    band_diff, outside, errs, secs, done = 0, 0, [], 0.0, 0
    for l in range(n_layers):
        OL = host_oracle_layer(stack.layers[l])
        x_before = xr.cpu().double().numpy()
        pi.pi_ffn_stack(pi.layer_array([stack.arr[l]]), xr, 1, idx, cnt, stack.ws)
        torch.cuda.synchronize()
        y_gpu = xr.cpu().double().numpy() - x_before
        g = idx[0, : int(cnt.item())].cpu().numpy()
        t0 = time.perf_counter()
        xl = oracle.rms_cast(x_before, cfg.adtype)
        _, I_or, s_or = oracle.sparse_ffn_layer(OL, xl)
        secs += time.perf_counter() - t0
        done += 1
        diff = np.setxor1d(g, I_or)
        inband = oracle.band(s_or, OL.threshold).any(axis=0)[diff]
        band_diff += int(inband.sum())
        outside += int((~inband).sum())
        y_or = oracle.masked_ffn(OL, xl, g)
        errs.append(float(np.linalg.norm(y_gpu - y_or) / np.linalg.norm(y_or)))
        del OL
        if secs >= budget_s and done >= 1:
            break
    tol = 2e-3 if cfg.wdtype == "q4_0" else 1e-3
    return {
        "layers": done, "token": 0,
        "index_mismatch_outside_band": outside,
        "band_neurons_excluded": band_diff,
        "max_rel_l2": float(f"{max(errs):.3e}"), "tol": tol,
        "ok": outside == 0 and max(errs) <= tol,
    }, secs / done, done


def run_ours(args, rank, world, local):
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
        cfg = dataclasses.replace(cfg, n_layers=min(args.layers, cfg.n_layers))
    B, T, NL, d, F = args.batch, cfg.n_tokens, cfg.n_layers, cfg.d_model, cfg.d_ff
    T = max(B, T // B * B)  # whole batches: a batch that does not divide the tokens drops the rest
    peak, peak_kind = measured_hbm()

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    # ---- headline: the stack generated on this GPU, graph replay of the step
    st = Stack(cfg, args.mode, B, world)
    X0 = st.tokens(T)
    Xw = torch.empty_like(X0)
    g, launches_per_step = st.graph(st.arr, X0, Xw)
    dev_id = "GPU-" + str(torch.cuda.get_device_properties(local).uuid)
    for _ in range(args.warmup):
        g.replay()
    torch.cuda.synchronize()
    with ClockSampler(dev_id) as clk:
        ms = st.time_graph(g, args.steps, 0, barrier)
    clocks = clk.summary()
    assert pi.pi_device_error() == 0, "device-side error flagged during the timed region"
    value = job_value(args.steps * T, world, ms)
    assert torch.isfinite(Xw).all()
    del g

    roofline, Ks, fb, durs = st.ffn_roofline(X0, Xw, peak)
    roofline["peak_kind"] = peak_kind
    if (TRAFFIC and TRAFFIC["src_sha"] == src_sha(TRAFFIC["files"]) and TRAFFIC["config"] == cfg.name
            and B == 1):
        roofline["traffic"] = round(TRAFFIC["ratio"] * roofline["algorithmic_bytes_per_launch"])
        roofline["traffic_source"] = TRAFFIC["profile"]
    else:
        roofline["traffic"] = None
    sb = st.step_bytes(fb.sum(), X0.shape[0])
    step_s = ms / args.steps / 1e3
    stack_roof = {"achieved": round(sb / step_s / 1e9, 1), "unit": "GB/s", "peak": peak,
                  "frac": round(sb / step_s / 1e9 / peak, 4),
                  "frac_of_nominal_8tbs": round(sb / step_s / 1e9 / NOMINAL_HBM_GBS, 4),
                  "bytes_per_step": round(sb)}
    if args.counts_out and rank == 0:
        with open(args.counts_out, "w") as f:
            json.dump({"order": "token-major, then layer", "counts": Ks.tolist(),
                       "algorithmic_bytes": fb.tolist(),
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
            pi.pi_sparse_ffn(st.arr[l], x16, B, idx_all, cnt_all, y, st.ws)
        torch.cuda.synchronize()
        gd = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gd):
            for t in range(T // B):
                for l in range(NL):
                    pi.pi_sparse_ffn(st.arr[l], x16, B, idx_all, cnt_all, y, st.ws)
        dreps = 2
        dms = st.time_graph(gd, dreps, 1, barrier)
        dense_tps = job_value(dreps * T, world, dms)
        extras["dense"] = {"value": round(dense_tps, 2), "unit": UNIT,
                           "speedup_sparse_over_dense": round(value / dense_tps, 3)}
        del gd

        # ---- mode F: same weights, predictor calibrated to the firing fraction
        other = "F" if args.mode == "R" else "R"
        layers_o = [synth.with_mode(L, other) for L in st.layers]  # keeps their b2 alive
        arr_o = st.descs(layers_o)
        go, _ = st.graph(arr_o, X0, Xw)
        osteps = max(3, args.steps // 2)
        oms = st.time_graph(go, osteps, 1, barrier)
        cnt_o = torch.zeros(NL, dtype=torch.int32, device="cuda")
        Xw.copy_(X0)
        pi.pi_ffn_stack(arr_o, Xw[0], B, None, cnt_o, st.ws)
        extras["mode_" + other] = {
            "value": round(job_value(osteps * T, world, oms), 2), "unit": UNIT,
            "mean_active_frac_token0": round(float(cnt_o.float().mean()) / F, 4)}
        del go, arr_o, layers_o

        # ---- e2e: public API, eager, host buffers in and out every step
        Xh = X0.cpu().pin_memory()
        Oh = torch.empty_like(Xh).pin_memory()

        def e2e_step():
            Xw.copy_(Xh, non_blocking=True)
            for t in range(T // B):
                pi.pi_ffn_stack(st.arr, Xw[t], B, None, None, st.ws)
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
        extras["e2e"] = {"value": round(job_value(esteps * T, world, ems), 2), "unit": UNIT,
                         "h2d_bytes_per_step": nbytes, "d2h_bytes_per_step": nbytes,
                         "steps": esteps, "api": "pi_ffn_stack per token, eager launches"}

        # ---- the prompt as one union step (the configs that have one)
        if cfg.prompt_tokens and B == 1:
            pst = st.with_batch(cfg.prompt_tokens)
            r, _, _ = measure(pst, cfg.prompt_tokens, 3, 1, peak, barrier, seed_offset=4242)
            r["config"] = workload_config(cfg, args.mode, pst.B, tokens=cfg.prompt_tokens)
            r["config"]["workload"] = r["config"]["workload"].replace("decode tokens per step",
                                                                      "prompt tokens per step")
            extras[f"prompt_b{pst.B}"] = r
            del pst

        # ---- parity sample and the oracle on the host (rank 0 of a 1-GPU run)
        if rank == 0 and world == 1:
            ps, per_layer, nl_done = parity_and_cpu_sample(
                st, X0[0, 0].cpu(), min(NL, SAMPLE_LAYERS), args.cpu_seconds)
            extras["parity_sample"] = ps
            hi = host_info()
            extras["cpu_baseline"] = {
                "value": round(1.0 / (per_layer * NL), 6), "unit": UNIT, "cores": 1,
                "kind": "oracle", "threads": 1, **hi,
                "sample": (f"token 0 of the workload through layers 0-{nl_done - 1} of {NL}, "
                           f"single-threaded C++ fp64 oracle, {per_layer:.3f} s per layer; "
                           f"tokens/s scaled to the {NL}-layer stack")}
        # ---- hot-row ordering: the same stack renumbered hottest-first
        if world == 1:
            hst = st.hot_first()
            r, _, _ = measure(hst, T, max(3, args.steps // 2), 1, peak)
            r["speedup_over_profile_order"] = round(r["value"] / value, 4)
            extras["hot_first"] = r
            del hst
    del st, X0, Xw
    torch.cuda.empty_cache()

    # ---- the other workloads, each on the first layers of its stack
    configs = {}
    if not args.no_extras and world == 1:
        for key, name, b, nl in EXTRAS:
            c = synth.get_config(name)
            c = dataclasses.replace(c, n_layers=min(nl, c.n_layers))
            s2 = Stack(c, args.mode, b, world)
            r, _, _ = measure(s2, c.n_tokens, 3, 1, peak)
            r["config"] = workload_config(c, args.mode, b)
            r["tokens_per_s_scaled_to_full_stack"] = round(
                r["value"] * c.n_layers / synth.get_config(name).n_layers, 2)
            configs[key] = r
            del s2
            torch.cuda.empty_cache()

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": cfg.wdtype,
            "data": "synthetic", "config": workload_config(cfg, args.mode, B, tokens=T),
            "roofline": roofline, "stack_roofline": stack_roof,
            "gpu_launches": int(launches_per_step * args.steps),
            "clocks": clocks,
        }
        for k in ("cpu_baseline", "e2e"):
            if k in extras:
                line[k] = extras.pop(k)
        line.update(extras)
        if configs:
            line["configs"] = configs
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


# ------------------------------------------------------------- reference arm
def run_reference(args, rank, world, local):
    """The single-threaded fp64 C++ oracle on the host.  Each step is one layer
    of the stack for token 0 of the workload, cycling over the same first layers
    the ours-arm CPU sample uses, with the residual stream carried."""
    if rank != 0:
        return
    import torch

    import oracle
    import synth

    cfg = synth.get_config(args.config)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    if dev == "cuda":
        torch.cuda.set_device(local)
    nl = min(cfg.n_layers, SAMPLE_LAYERS)
    hosts = []
    for l in range(nl):
        hosts.append(host_oracle_layer(synth.make_layer(cfg, l, dev, args.mode)))
        if dev == "cuda":
            torch.cuda.empty_cache()
    x = synth.make_tokens(cfg, args.batch).double().numpy()
    times = []
    for s in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        xl = oracle.rms_cast(x, cfg.adtype)
        y, _, _ = oracle.sparse_ffn_layer(hosts[s % nl], xl)
        x = x + y
        dt = time.perf_counter() - t0
        if s >= args.warmup:
            times.append(dt)
    per_layer = sum(times) / len(times)
    value = args.batch / (per_layer * cfg.n_layers)
    sample = (f"each step: one of layers 0-{nl - 1} of {cfg.n_layers} (in turn) for token 0 of "
              f"the workload, single-threaded C++ fp64 oracle; tokens/s scaled to the "
              f"{cfg.n_layers}-layer stack")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(per_layer * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(cfg, args.mode, args.batch),
        "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": 1, "kind": "oracle",
                         "threads": 1, **host_info(), "sample": sample},
        "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0,
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
