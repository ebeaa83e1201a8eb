#!/usr/bin/env python3
"""Benchmark of the BitLinear forward on a BitNet b1.58 2B4T-shaped layer stack.

Workload (one "step"): all BitLinear projections of 30 random-init layers
(hidden 2560, intermediate 6912): q and o (2560 -> 2560), the fused gate/up
FFN (2560 -> 2 x 6912, relu(gate)^2 * up) and down (6912 -> 2560).  A step is
one prefill pass over 8 x 512 = 4096 tokens followed by 128 decode steps at
batch 8, every projection through the library's C ABI (Python binding), each
phase captured once as CUDA graphs and replayed.  Weights are ternarised and
packed once before timing (the method does this offline).

Reported metric: BitLinear throughput as tokens/s per layer (token-layers per
second of device time; prefill and decode tokens both count), with the phase
breakdown in GB/s (decode, against HBM) and TOPS (prefill, against the int8
tensor-core peak), a roofline entry for the kernel with the largest share of
the step, the oracle timed on the host, and an end-to-end figure with
host<->device copies inside the timed region.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (torchrun, one process per GPU) every rank runs its own replica on
its own batch (data parallel, no collective on the data path; weak scaling);
the time is the max over ranks.
"""
import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "BitLinear GB/s and TOPS (% of HBM / INT8 roofline); decode tokens/s per layer"
UNIT = "tokens/s per layer"
HIDDEN, INTER = 2560, 6912
QKV = HIDDEN + 2 * 640  # fused q, k, v projection of the grouped-query attention (k / v: 2560 -> 640)
NOMINAL_INT8_PER_BF16 = 2.0  # dense int8 / dense bf16 tensor rate on B200 (4.5 / 2.25 PFLOP/s)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=10)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--layers", type=int, default=30)
    p.add_argument("--prefill-tokens", type=int, default=4096)
    p.add_argument("--decode-steps", type=int, default=128)
    p.add_argument("--decode-batch", type=int, default=8)
    p.add_argument("--e2e-steps", type=int, default=None,
                   help="steps of the end-to-end measurement (default: --steps; 0 skips it)")
    p.add_argument("--cpu-seconds", type=float, default=10.0, help="budget of the oracle CPU baseline")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-configs", action="store_true",
                   help="skip the single-BitLinear and FFN lines at decode sizes (configs 2 and 3)")
    p.add_argument("--decode-path", choices=["sequence", "per-op"], default="sequence",
                   help="decode step as one persistent bitnet_decode_sequence launch (default) or one "
                        "bitnet_linear / bitnet_ffn_gate_up call per projection")
    p.add_argument("--profile", default=None,
                   choices=["decode_q_o", "decode_gate_up", "decode_down", "prefill_q_o", "prefill_gate_up",
                            "prefill_down", "decode_sequence"],
                   help="profiling harness: build one layer, run this projection kind --profile-reps times "
                        "(no graphs, no timing, no JSON) and exit; for ncu captures of one kernel")
    p.add_argument("--profile-reps", type=int, default=3)
    a = p.parse_args()
    if a.e2e_steps is None:
        a.e2e_steps = a.steps
    return a


def workload_config(a, n_gpus):
    return {
        "workload": (f"bitnet-b1.58-2b4t BitLinear stack: {a.layers} layers x (q, o {HIDDEN}x{HIDDEN}; "
                     f"gate/up {HIDDEN}->2x{INTER} + relu2; down {INTER}->{HIDDEN}); "
                     f"prefill {a.prefill_tokens} tokens (8x512) then {a.decode_steps} decode steps at batch "
                     f"{a.decode_batch}"),
        "layers": a.layers, "hidden": HIDDEN, "intermediate": INTER,
        "prefill_tokens": a.prefill_tokens, "decode_steps": a.decode_steps, "decode_batch": a.decode_batch,
        "activations": "bf16 N(0,1), fresh per projection; ternary weights from N(0,0.02) latents",
        "decode_path": a.decode_path,
        "decode_outputs": "one set per layer",
        "l2": "inputs larger than L2: every pass streams 496 MB of packed weights; prefill activations rotate "
              "over 168 MB",
        "parallelism": f"replicas x{n_gpus} (data parallel, no collective)",
    }


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ oracle (CPU)
def oracle_layer_sample(tokens, seed=4242):
    """Bounded CPU sample of the workload: `tokens` tokens through one layer's
    four projections with the oracle.  Returns (closure, description)."""
    import numpy as np

    import oracle
    sys.path.insert(0, os.path.join(os.path.dirname(os.path.abspath(__file__)), "tests"))
    import synth  # the seeded input generators shared with the tests

    mats = {}
    for j, (name, n, k) in enumerate((("q", HIDDEN, HIDDEN), ("o", HIDDEN, HIDDEN), ("gate", INTER, HIDDEN),
                                      ("up", INTER, HIDDEN), ("down", HIDDEN, INTER))):
        p, g, _ = oracle.pack_weights(synth.latent_weights(n, k, seed + j))
        mats[name] = (p, g, k)
    xs = [synth.bf16_bits_to_f32(synth.activations(tokens, HIDDEN, seed + 10 + i)) for i in range(3)]

    def run():
        oracle.bitlinear(xs[0], *mats["q"])
        oracle.bitlinear(xs[1], *mats["o"])
        h = oracle.ffn_gate_up(xs[2], mats["gate"][0], mats["gate"][1], mats["up"][0], mats["up"][1], HIDDEN)[0]
        oracle.bitlinear(h.astype(np.float32), *mats["down"])

    return run, (f"{tokens} tokens through one layer (q, o, gate/up+relu2, down) with the C oracle, "
                 f"single thread; tokens/s per layer = tokens / time")


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


_WORKER_RUN = []


def _oracle_init(tokens, seed):
    """Pool initializer: pack the one-layer oracle sample's weights once per worker process."""
    _WORKER_RUN.append(oracle_layer_sample(tokens, seed=seed)[0])


def _oracle_worker(reps):
    """One pool task: `reps` passes of the worker's oracle sample; returns its run time."""
    run = _WORKER_RUN[0]
    t0 = time.perf_counter()
    for _ in range(reps):
        run()
    return time.perf_counter() - t0


def cpu_baseline(budget_s, tokens=8):
    """The oracle as it stands, on the host: single-threaded, then one independent copy per host core
    (a spawn-started process pool; the oracle itself is unchanged and single-threaded)."""
    run, desc = oracle_layer_sample(tokens)
    run()  # warm
    times = []
    t_end = time.perf_counter() + budget_s / 2
    while time.perf_counter() < t_end or len(times) < 2:
        t0 = time.perf_counter()
        run()
        times.append(time.perf_counter() - t0)
    single = tokens / statistics.mean(times)
    cores = os.cpu_count() or 1
    out = {"value": single, "unit": UNIT, "cores": 1, "kind": "oracle",
           "sample": f"{desc}; {len(times)} repetitions, {sum(times):.1f} s",
           "host_cores": cores, "cpu_model": cpu_model()}
    if cores > 1:
        import multiprocessing as mp
        reps = max(1, int(budget_s / 2 / statistics.mean(times)))
        try:
            with mp.get_context("spawn").Pool(cores, initializer=_oracle_init, initargs=(tokens, 4242)) as pool:
                pool.map(_oracle_worker, [0] * cores, chunksize=1)  # every worker started and packed, untimed
                t0 = time.perf_counter()
                pool.map(_oracle_worker, [reps] * cores, chunksize=1)
                wall = time.perf_counter() - t0
            out["value"] = cores * reps * tokens / wall
            out["cores"] = cores
            out["sample"] = (f"{desc.replace('single thread', f'{cores} processes (one per host core)')}; "
                             f"{reps} repetitions per process, {wall:.1f} s wall")
            out["single_thread"] = {"value": single, "cores": 1}
        except Exception as e:  # noqa: BLE001 - the single-thread figure stands
            out["all_cores_error"] = f"{type(e).__name__}: {e}"
    return out


def reference_arm(a, n_gpus):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    tokens = a.decode_batch
    run, desc = oracle_layer_sample(tokens)
    for _ in range(a.warmup):
        run()
    times = []
    for _ in range(a.steps):
        t0 = time.perf_counter()
        run()
        times.append(time.perf_counter() - t0)
    ms = 1e3 * statistics.mean(times)
    value = tokens / (ms / 1e3)
    cfg = workload_config(a, n_gpus)
    cfg["sample"] = desc
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": n_gpus,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int64", "data": "synthetic", "config": cfg,
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.out, stderr=subprocess.DEVNULL)
        except (OSError, ValueError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------ configs 2 and 3
def check_context(torch, tw, where):
    """Raise if the CUDA context holds a sticky error or a device-side wait gave up: numbers taken
    after that would come from a broken context."""
    torch.cuda.synchronize()
    stat = tw.bitnet_device_status(clear=False)
    if stat != 0:
        raise RuntimeError(f"{where}: device status {tw.bitnet_status_string(stat)}")


def decode_configs(st, stream, hbm_peak, l2_bytes):
    """Single BitLinears and FFNs at decode sizes, each timed two ways (CUDA events over a CUDA graph):
      per_op    one bitnet_linear / bitnet_ffn_gate_up call per projection, consecutive calls rotating
                over distinct weight copies (>= 3 x L2 of weights), so every call streams from HBM;
      sequence  the same projections as independent ops of one bitnet_decode_sequence launch.
    GEMV at M = 1: 2560 -> 2560, 2560 -> 6912, 6912 -> 2560.  FFN at M in {1, 8, 16, 32, 64}: gate/up
    2560 -> 2 x 6912 with relu(gate)^2 * up, then down 6912 -> 2560 on its h (the stack's 30 layers of
    weights, 398 MB).  Bytes = packed weights + activations in + outputs."""
    torch, tw = st.torch, st.tw
    dev = st.dev
    f32 = torch.float32
    out = {"gemv_m1": {}, "ffn": {}}

    def timed(fn, n_calls, reps=5):
        g = capture(torch, stream, fn)
        ms = time_graph(torch, stream, g, reps)
        del g
        return ms / n_calls

    def line(us, nbytes, tokens=None):
        gbs = nbytes / (us / 1e6) / 1e9
        d = {"us": us, "bytes": nbytes, "gbs": gbs, "frac_hbm": gbs / hbm_peak}
        if tokens is not None:
            d["tokens_per_s"] = tokens / (us / 1e6)
        return d

    with torch.cuda.stream(stream):
        # ---- config 2: GEMV at M = 1 ----
        x1 = torch.randn((1, INTER), generator=st.gen, device=dev).to(torch.bfloat16)
        for (k, n) in ((HIDDEN, HIDDEN), (HIDDEN, INTER), (INTER, HIDDEN)):
            lat = torch.randn((n, k), generator=st.gen, device=dev, dtype=f32).mul_(0.02)
            p0, g0 = tw.bitnet_pack_weights(lat)
            del lat
            wbytes = n * k // 4
            copies = max(128, -(-3 * l2_bytes // wbytes))
            ws = torch.empty(copies * wbytes, dtype=torch.uint8, device=dev).view(copies, n, k // 4)
            ws.copy_(p0.unsqueeze(0).expand(copies, n, k // 4))
            x = x1[:, :k].contiguous()
            ys = torch.empty((copies, 1, n), dtype=f32, device=dev)
            wsp = torch.empty(tw.bitnet_workspace_size(1, n, k), dtype=torch.uint8, device=dev)
            per_call = wbytes + k * 2 + n * 4
            us = timed(lambda s: [tw.bitnet_linear(x, ws[c], g0, y=ys[c], workspace=wsp, stream=s)
                                  for c in range(copies)], copies) * 1e3
            key = f"{k}x{n}"
            out["gemv_m1"][key] = {"per_op": line(us, per_call), "copies": copies}
            # one launch of 128 independent GEMVs (two alternating halves of the copies)
            nseq = 128
            halves = [[tw.linear_op(x, ws[(h * nseq + c) % copies], g0, ys[(h * nseq + c) % copies])
                       for c in range(nseq)] for h in range(2)]
            wsq = tw.bitnet_sequence_workspace(dev, nseq, 1, k)
            us = timed(lambda s: [tw.bitnet_decode_sequence(halves[r % 2], 1, wsq, stream=s) for r in range(4)],
                       4) * 1e3
            out["gemv_m1"][key]["sequence"] = line(us / nseq, per_call)
            out["gemv_m1"][key]["sequence"]["ops_per_launch"] = nseq
            del ws, ys, wsq
            check_context(torch, tw, f"gemv {key}")
        # ---- config 3: FFN (gate/up + down) at M in {1, 8, 16, 32, 64} ----
        L = st.layers
        nl = len(L)
        for m in (1, 8, 16, 32, 64):
            xs = [torch.randn((m, HIDDEN), generator=st.gen, device=dev).to(torch.bfloat16) for _ in range(nl)]
            hs = [torch.empty((m, INTER), dtype=f32, device=dev) for _ in range(nl)]
            ds = [torch.empty((m, HIDDEN), dtype=f32, device=dev) for _ in range(nl)]
            wsp = torch.empty(tw.bitnet_workspace_size(m, INTER, INTER), dtype=torch.uint8, device=dev)
            per_ffn = 3 * INTER * HIDDEN // 4 + m * HIDDEN * 2 + 2 * m * INTER * 4 + m * HIDDEN * 4

            def per_op(s):
                for l in range(nl):
                    tw.bitnet_ffn_gate_up(xs[l], L[l]["gate"][0], L[l]["gate"][1], L[l]["up"][0], L[l]["up"][1],
                                          h=hs[l], workspace=wsp, stream=s)
                    tw.bitnet_linear(hs[l], L[l]["down"][0], L[l]["down"][1], y=ds[l], workspace=wsp, stream=s)
            us = timed(per_op, nl) * 1e3
            ops = []
            for l in range(nl):
                ops += [tw.ffn_gate_up_op(xs[l], L[l]["gate"][0], L[l]["gate"][1], L[l]["up"][0], L[l]["up"][1],
                                          hs[l]),
                        tw.linear_op(hs[l], L[l]["down"][0], L[l]["down"][1], ds[l])]
            wsq = tw.bitnet_sequence_workspace(dev, len(ops), m, INTER)
            us_seq = timed(lambda s: [tw.bitnet_decode_sequence(ops, m, wsq, stream=s) for _ in range(3)], 3) * 1e3
            out["ffn"][f"M={m}"] = {"per_op": line(us, per_ffn, m), "sequence": line(us_seq / nl, per_ffn, m)}
            out["ffn"][f"M={m}"]["sequence"]["ffns_per_launch"] = nl
            del xs, hs, ds, wsp, wsq
            check_context(torch, tw, f"ffn M={m}")
    return out


# ------------------------------------------------------------------ our arm
class Stack:
    """Packed weights, activation pools and output buffers of the layer stack."""

    def __init__(self, a, device, seed):
        import torch

        import ternary_weight_fwd_b200 as tw

        self.a, self.dev, self.tw, self.torch = a, device, tw, torch
        gen = torch.Generator(device=device)
        gen.manual_seed(seed)
        self.layers = []
        for _ in range(a.layers):
            layer = {}
            for name, n, k in (("q", HIDDEN, HIDDEN), ("o", HIDDEN, HIDDEN), ("gate", INTER, HIDDEN),
                               ("up", INTER, HIDDEN), ("down", HIDDEN, INTER)):
                w = torch.randn((n, k), generator=gen, device=device, dtype=torch.float32).mul_(0.02)
                layer[name] = tw.bitnet_pack_weights(w)
                del w
            self.layers.append(layer)
        torch.cuda.synchronize()
        M, B = a.prefill_tokens, a.decode_batch
        self.n_pre = 8   # 8 x 21 MB of bf16 prefill activations (> L2) rotated over the projections
        self.n_dec = 64
        self.pre_x = [torch.randn((M, HIDDEN), generator=gen, device=device).to(torch.bfloat16)
                      for _ in range(self.n_pre)]
        self.dec_x = [torch.randn((B, HIDDEN), generator=gen, device=device).to(torch.bfloat16)
                      for _ in range(self.n_dec)]
        f32 = torch.float32
        self.pre_out = {"q": torch.empty((M, HIDDEN), dtype=f32, device=device),
                        "o": torch.empty((M, HIDDEN), dtype=f32, device=device),
                        "h": torch.empty((M, INTER), dtype=f32, device=device),
                        "down": torch.empty((M, HIDDEN), dtype=f32, device=device)}
        self.dec_out = {"q": torch.empty((B, HIDDEN), dtype=f32, device=device),
                        "o": torch.empty((B, HIDDEN), dtype=f32, device=device),
                        "h": torch.empty((B, INTER), dtype=f32, device=device),
                        "down": torch.empty((B, HIDDEN), dtype=f32, device=device)}
        # the decode step's outputs, one set per layer: the layers of a step share no buffers, so the
        # only dependency inside a step is gate/up -> down of each layer (fresh x for every other op)
        self.dec_out_l = [{"q": torch.empty((B, HIDDEN), dtype=f32, device=device),
                           "o": torch.empty((B, HIDDEN), dtype=f32, device=device),
                           "h": torch.empty((B, INTER), dtype=f32, device=device),
                           "down": torch.empty((B, HIDDEN), dtype=f32, device=device)} for _ in range(a.layers)]
        ws = max(tw.bitnet_workspace_size(M, n, k) for n, k in ((HIDDEN, HIDDEN), (INTER, HIDDEN), (HIDDEN, INTER),
                                                                 (QKV, HIDDEN)))
        self.ws_pre = torch.empty(ws, dtype=torch.uint8, device=device)
        self.ws_dec = torch.empty(tw.bitnet_workspace_size(B, INTER, INTER), dtype=torch.uint8, device=device)
        self.ws_seq = tw.bitnet_sequence_workspace(device, 4 * a.layers, B, INTER)
        self.norm_g = (torch.randn(HIDDEN, generator=gen, device=device) * 0.1 + 1.0).float()
        self.q_buf = torch.empty((M, HIDDEN), dtype=torch.int8, device=device)
        self.s_buf = torch.empty(M, dtype=torch.float32, device=device)
        self.rs_buf = torch.empty(M, dtype=torch.int32, device=device)
        self.gen = gen
        # bf16 gate/up -> down chain through the emitted per-token maxima of h
        bf = torch.bfloat16
        self.pre_hb = torch.empty((M, INTER), dtype=bf, device=device)
        self.pre_db = torch.empty((M, HIDDEN), dtype=bf, device=device)
        self.pre_ha = torch.empty(M, dtype=f32, device=device)
        self.dec_hb = torch.empty((B, INTER), dtype=bf, device=device)
        self.dec_db = torch.empty((B, HIDDEN), dtype=bf, device=device)
        self.dec_ha = torch.empty(B, dtype=f32, device=device)
        self.seq_ops = {}
        self.packed_bytes = sum(L[k][0].numel() for L in self.layers for k in ("q", "o", "gate", "up", "down"))

    # one projection of each kind -------------------------------------------
    def q(self, l, x, out, ws, s):
        L = self.layers[l]
        self.tw.bitnet_linear(x, L["q"][0], L["q"][1], y=out["q"], workspace=ws, stream=s)

    def o(self, l, x, out, ws, s):
        L = self.layers[l]
        self.tw.bitnet_linear(x, L["o"][0], L["o"][1], y=out["o"], workspace=ws, stream=s)

    def gate_up(self, l, x, out, ws, s):
        L = self.layers[l]
        self.tw.bitnet_ffn_gate_up(x, L["gate"][0], L["gate"][1], L["up"][0], L["up"][1], h=out["h"],
                                   workspace=ws, stream=s)

    def down(self, l, out, ws, s):
        L = self.layers[l]
        self.tw.bitnet_linear(out["h"], L["down"][0], L["down"][1], y=out["down"], workspace=ws, stream=s)

    def ensure_qkv(self):
        """Fused QKV projection weights and outputs, made only when those kinds are timed (after the
        step), so the step's launch sequence does not change."""
        if hasattr(self, "pre_qkv"):
            return
        torch, tw = self.torch, self.tw
        for layer in self.layers:
            w = torch.randn((QKV, HIDDEN), generator=self.gen, device=self.dev, dtype=torch.float32).mul_(0.02)
            layer["qkv"] = tw.bitnet_pack_weights(w)
            del w
        self.dec_qkv = torch.empty((self.a.decode_batch, QKV), dtype=torch.float32, device=self.dev)
        self.pre_qkv = torch.empty((self.a.prefill_tokens, QKV), dtype=torch.float32, device=self.dev)
        torch.cuda.synchronize()

    def qkv(self, l, x, out, ws, s):
        L = self.layers[l]
        self.tw.bitnet_linear(x, L["qkv"][0], L["qkv"][1], y=out, workspace=ws, stream=s)

    def ffn_bf16_chain(self, l, x, hb, ha, db, ws, s):
        """gate/up with bf16 h and its emitted maxima, then down fed those maxima."""
        L, tw = self.layers[l], self.tw
        tw.bitnet_ffn_gate_up_ex(x, L["gate"][0], L["gate"][1], L["up"][0], L["up"][1], h=hb, h_amax=ha,
                                 workspace=ws, stream=s)
        tw.bitnet_linear_ex(hb, L["down"][0], L["down"][1], x_amax=ha, y=db, workspace=ws, stream=s)

    def prefill_pass(self, s):
        for l in range(self.a.layers):
            self.q(l, self.pre_x[(3 * l) % self.n_pre], self.pre_out, self.ws_pre, s)
            self.o(l, self.pre_x[(3 * l + 1) % self.n_pre], self.pre_out, self.ws_pre, s)
            self.gate_up(l, self.pre_x[(3 * l + 2) % self.n_pre], self.pre_out, self.ws_pre, s)
            self.down(l, self.pre_out, self.ws_pre, s)

    def decode_ops(self, t):
        """The projections of decode step t as bitnet_op_t records (one sequence launch)."""
        if t not in self.seq_ops:
            tw, ops = self.tw, []
            for l in range(self.a.layers):
                L, out = self.layers[l], self.dec_out_l[l]
                base = t * 3 * self.a.layers + 3 * l
                ops += [tw.linear_op(self.dec_x[base % self.n_dec], L["q"][0], L["q"][1], out["q"]),
                        tw.linear_op(self.dec_x[(base + 1) % self.n_dec], L["o"][0], L["o"][1], out["o"]),
                        tw.ffn_gate_up_op(self.dec_x[(base + 2) % self.n_dec], L["gate"][0], L["gate"][1],
                                          L["up"][0], L["up"][1], out["h"]),
                        tw.linear_op(out["h"], L["down"][0], L["down"][1], out["down"])]
            self.seq_ops[t] = ops
        return self.seq_ops[t]

    def decode_step(self, t, s):
        if self.a.decode_path == "sequence":
            self.tw.bitnet_decode_sequence(self.decode_ops(t), self.a.decode_batch, self.ws_seq, stream=s)
            return
        for l in range(self.a.layers):
            base = t * 3 * self.a.layers + 3 * l
            out = self.dec_out_l[l]
            self.q(l, self.dec_x[base % self.n_dec], out, self.ws_dec, s)
            self.o(l, self.dec_x[(base + 1) % self.n_dec], out, self.ws_dec, s)
            self.gate_up(l, self.dec_x[(base + 2) % self.n_dec], out, self.ws_dec, s)
            self.down(l, out, self.ws_dec, s)


def reduce_max(v, dist, device):
    """Max of a float over all ranks (identity without a process group)."""
    if dist is None:
        return v
    import torch

    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_value(n_gpus, tokens_per_replica_step, layers, max_ms_per_step):
    """Whole-job throughput: every replica processes its own batch (weak scaling)."""
    return n_gpus * tokens_per_replica_step * layers / (max_ms_per_step / 1e3)


def capture(torch, stream, fn):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn(stream)
    return g


def time_graph(torch, stream, graph, reps):
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        graph.replay()
        stream.synchronize()
        e0.record(stream)
        for _ in range(reps):
            graph.replay()
        e1.record(stream)
    e1.synchronize()
    return e0.elapsed_time(e1) / reps


# The sources each measured kernel family is built from (its device code, the headers that code
# includes, and the host code that plans and launches it); include/bitnet.h is always added.
KIND_SOURCES = {
    "decode_sequence": ["bitnet.cu", "common.cuh", "decode.cuh", "decode_tasks.cuh", "exact_sumsq.cuh",
                        "pack_quant.cuh"],
    "prefill": ["bitnet.cu", "common.cuh", "pack_quant.cuh", "prefill.cuh"],
}


def strip_comments(src):
    """C/C++ source without comments and blank lines (string and character literals kept)."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c in "\"'":
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    return "\n".join(l.rstrip() for l in "".join(out).splitlines() if l.strip())


def source_digest(kind=None):
    """sha256 (first 16 hex digits) of the code of the kernel sources of `kind` (all of csrc/ when
    None); comments do not count, so a documentation change keeps counters taken on the same code."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "ternary_weight_fwd_b200", "csrc")
    files = sorted(os.listdir(csrc))
    if kind is not None:
        files = sorted(KIND_SOURCES["prefill" if kind.startswith("prefill") else kind])
    paths = [os.path.join(csrc, f) for f in files] + [os.path.join(ROOT, "include", "bitnet.h")]
    for path in paths:
        with open(path, encoding="utf-8") as fh:
            h.update(os.path.basename(path).encode())
            h.update(strip_comments(fh.read()).encode())
    return h.hexdigest()[:16]


def dram_traffic(kernel_key):
    """Per-launch DRAM bytes of a kernel from the committed ncu summary, if it was
    taken on the current kernel sources; otherwise None."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    e = d.get(kernel_key)
    if not e or e.get("source_digest") != source_digest(kernel_key):
        return None
    return e.get("bytes_per_launch")


def our_arm(a, n_gpus):
    import torch

    import ternary_weight_fwd_b200 as tw
    from ternary_weight_fwd_b200 import build as tw_build

    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    dist = None
    if world > 1:
        import torch.distributed as dist_mod
        dist = dist_mod
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    if rank == 0:
        tw_build.build()
    if dist:
        dist.barrier()
    tw.load_library()
    peaks, peaks_src = load_peaks()

    def barrier():
        if dist:
            dist.barrier()

    def max_over_ranks(v):
        return reduce_max(v, dist, dev)

    st = Stack(a, dev, seed=1234 + rank)
    stream = torch.cuda.Stream(device=dev)
    stream.wait_stream(torch.cuda.current_stream())

    if a.profile:
        ops = {
            "decode_q_o": lambda s: st.q(0, st.dec_x[0], st.dec_out, st.ws_dec, s),
            "decode_gate_up": lambda s: st.gate_up(0, st.dec_x[0], st.dec_out, st.ws_dec, s),
            "decode_down": lambda s: st.down(0, st.dec_out, st.ws_dec, s),
            "prefill_q_o": lambda s: st.q(0, st.pre_x[0], st.pre_out, st.ws_pre, s),
            "prefill_gate_up": lambda s: st.gate_up(0, st.pre_x[0], st.pre_out, st.ws_pre, s),
            "prefill_down": lambda s: st.down(0, st.pre_out, st.ws_pre, s),
            "decode_sequence": lambda s: st.decode_step(0, s),
        }
        with torch.cuda.stream(stream):
            for _ in range(a.profile_reps):
                ops[a.profile](stream)
        stream.synchronize()
        assert tw.bitnet_device_status() == 0
        print(f"profiled {a.profile} x{a.profile_reps}")
        return 0

    # ---- capture: one prefill pass, decode steps in chunks of 16 ----
    with torch.cuda.stream(stream):
        c0 = tw.bitnet_launch_count()
        g_pre = capture(torch, stream, st.prefill_pass)
        c1 = tw.bitnet_launch_count()
        chunk = 16
        g_dec = []
        for t0 in range(0, a.decode_steps, chunk):
            g_dec.append(capture(torch, stream, lambda s, t0=t0: [st.decode_step(t, s) for t in
                                                                  range(t0, min(t0 + chunk, a.decode_steps))]))
        c2 = tw.bitnet_launch_count()
    launches_pre, launches_dec = c1 - c0, c2 - c1

    def run_step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        g_pre.replay()
        if ev is not None:
            ev[1].record(stream)
        for g in g_dec:
            g.replay()
        if ev is not None:
            ev[2].record(stream)

    # graphs replay on the current stream: keep `stream` current for every replay
    with torch.cuda.stream(stream):
        for _ in range(a.warmup):
            run_step()
        stream.synchronize()
        barrier()
        clocks = ClockSampler(local_rank if world > 1 else torch.cuda.current_device())
        clocks.start()
        time.sleep(0.3)
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(a.steps)]
        t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        barrier()
        t_start.record(stream)
        for i in range(a.steps):
            run_step(evs[i])
        t_end.record(stream)
        stream.synchronize()
    torch.cuda.synchronize()
    clk = clocks.stop()
    total_ms = max_over_ranks(t_start.elapsed_time(t_end))
    pre_ms = max_over_ranks(statistics.mean(e[0].elapsed_time(e[1]) for e in evs))
    dec_ms = max_over_ranks(statistics.mean(e[1].elapsed_time(e[2]) for e in evs))
    barrier()
    ms_step = total_ms / a.steps
    assert tw.bitnet_device_status() == 0, "a device-side wait timed out"

    M, B, Lyr = a.prefill_tokens, a.decode_batch, a.layers
    tokens_step = (M + a.decode_steps * B)
    value = aggregate_value(n_gpus, tokens_step, Lyr, ms_step)

    # ---- phase figures (per replica) ----
    ops_layer = 2 * HIDDEN * HIDDEN * 2 + 2 * (2 * HIDDEN * INTER) + 2 * INTER * HIDDEN  # per token
    pre_ops = M * Lyr * ops_layer
    pre_tops = pre_ops / (pre_ms / 1e3) / 1e12
    int8_peak_sust = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]) * \
        NOMINAL_INT8_PER_BF16
    int8_peak_burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]) * NOMINAL_INT8_PER_BF16
    pk_w = st.packed_bytes
    act_dec = Lyr * (B * HIDDEN * 2 * 3 + B * INTER * 4 + B * HIDDEN * 4 * 3 + B * INTER * 4)
    dec_bytes_step = pk_w + act_dec
    dec_step_ms = dec_ms / a.decode_steps
    dec_gbs = dec_bytes_step / (dec_step_ms / 1e3) / 1e9
    hbm_peak = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    phases = {
        "prefill_ms": pre_ms, "prefill_tops": pre_tops, "prefill_int8_peak_tops": int8_peak_sust,
        "prefill_frac_int8": pre_tops / int8_peak_sust,
        "prefill_tokens_per_s_per_layer": M * Lyr / (pre_ms / 1e3),
        "decode_ms_per_step": dec_step_ms, "decode_gbs": dec_gbs, "decode_frac_hbm": dec_gbs / hbm_peak,
        "decode_tokens_per_s_per_layer": B * Lyr / (dec_step_ms / 1e3),
        "peaks": (f"{peaks_src}: HBM {hbm_peak} GB/s; int8 of the prefill pass (a long phase) = sustained "
                  f"bf16 x {NOMINAL_INT8_PER_BF16}; int8 of a kind timed alone = burst bf16 x "
                  f"{NOMINAL_INT8_PER_BF16} = {int8_peak_burst:.0f} TOPS"),
    }

    # ---- per-kernel averages (CUDA events over graphs of one projection kind) ----
    # Every kind is timed; "in_step" marks the kinds the timed step runs (the decode
    # step is either one sequence launch or one call per projection).
    kinds = {}
    R = 4
    seq = a.decode_path == "sequence"
    with torch.cuda.stream(stream):
        specs = {
            "decode_sequence": (lambda s: [st.decode_step(t, s) for t in range(R)] if seq else None,
                                dec_bytes_step, "hbm", 1, R, seq),
            "decode_q_o": (lambda s: [st.q(l, st.dec_x[l % st.n_dec], st.dec_out, st.ws_dec, s)
                                      for _ in range(R) for l in range(Lyr)],
                           HIDDEN * HIDDEN // 4 + B * HIDDEN * 2 + B * HIDDEN * 4, "hbm", 2 * Lyr, R * Lyr, not seq),
            "decode_gate_up": (lambda s: [st.gate_up(l, st.dec_x[l % st.n_dec], st.dec_out, st.ws_dec, s)
                                          for _ in range(R) for l in range(Lyr)],
                               2 * INTER * HIDDEN // 4 + B * HIDDEN * 2 + B * INTER * 4, "hbm", Lyr, R * Lyr,
                               not seq),
            "decode_down": (lambda s: [st.down(l, st.dec_out, st.ws_dec, s) for _ in range(R) for l in range(Lyr)],
                            INTER * HIDDEN // 4 + B * INTER * 4 + B * HIDDEN * 4, "hbm", Lyr, R * Lyr, not seq),
            "prefill_q_o": (lambda s: [st.q(l, st.pre_x[l % st.n_pre], st.pre_out, st.ws_pre, s)
                                       for l in range(Lyr)], 2 * M * HIDDEN * HIDDEN, "tensor", 2 * Lyr, Lyr, True),
            "prefill_gate_up": (lambda s: [st.gate_up(l, st.pre_x[l % st.n_pre], st.pre_out, st.ws_pre, s)
                                           for l in range(Lyr)], 2 * 2 * M * HIDDEN * INTER, "tensor", Lyr, Lyr,
                                True),
            "prefill_down": (lambda s: [st.down(l, st.pre_out, st.ws_pre, s) for l in range(Lyr)],
                             2 * M * INTER * HIDDEN, "tensor", Lyr, Lyr, True),
            # the activation quantiser alone, and with the RMS normalisation fused in (not in the step)
            "prefill_quant": (lambda s: [tw.bitnet_quant_act(st.pre_x[l % st.n_pre], x_q=st.q_buf, s=st.s_buf,
                                                             rowsum=st.rs_buf, stream=s) for l in range(Lyr)],
                              M * HIDDEN * 2 + M * HIDDEN + 8 * M, "hbm", 0, Lyr, False),
            "prefill_rmsnorm_quant": (lambda s: [tw.bitnet_rmsnorm_quant(st.pre_x[l % st.n_pre], st.norm_g, x_q=st.q_buf,
                                                                         s=st.s_buf, rowsum=st.rs_buf, stream=s)
                                                 for l in range(Lyr)],
                                      M * HIDDEN * 2 + HIDDEN * 4 + M * HIDDEN + 8 * M, "hbm", 0, Lyr, False),
            # bf16 h with emitted maxima -> down fed them, against prefill_gate_up + prefill_down
            # (not in the step: the step stores fp32 outputs)
            "prefill_ffn_bf16_chain": (lambda s: [st.ffn_bf16_chain(l, st.pre_x[l % st.n_pre], st.pre_hb, st.pre_ha,
                                                                    st.pre_db, st.ws_pre, s) for l in range(Lyr)],
                                       2 * 2 * M * HIDDEN * INTER + 2 * M * INTER * HIDDEN, "tensor", 0, Lyr,
                                       False),
            "decode_ffn_bf16_chain": (lambda s: [st.ffn_bf16_chain(l, st.dec_x[l % st.n_dec], st.dec_hb, st.dec_ha,
                                                                   st.dec_db, st.ws_dec, s)
                                                 for _ in range(R) for l in range(Lyr)],
                                      3 * INTER * HIDDEN // 4 + B * HIDDEN * 2 + 2 * B * INTER * 2 + B * HIDDEN * 2,
                                      "hbm", 0, R * Lyr, False),
            # fused QKV BitLinear 2560 -> 3840 (q 2560 + k 640 + v 640), not in the step
            "decode_qkv": (lambda s: [st.qkv(l, st.dec_x[l % st.n_dec], st.dec_qkv, st.ws_dec, s)
                                      for _ in range(R) for l in range(Lyr)],
                           QKV * HIDDEN // 4 + B * HIDDEN * 2 + B * QKV * 4, "hbm", 0, R * Lyr, False),
            "prefill_qkv": (lambda s: [st.qkv(l, st.pre_x[l % st.n_pre], st.pre_qkv, st.ws_pre, s)
                                       for l in range(Lyr)], 2 * M * QKV * HIDDEN, "tensor", 0, Lyr, False),
        }
        for name, (fn, work, bound, per_step, n_ops, in_step) in specs.items():
            if name == "decode_sequence" and not seq:
                continue
            if not in_step:
                # kinds outside the step run once eagerly first: one that fails is reported, not fatal
                try:
                    if name.endswith("_qkv"):
                        st.ensure_qkv()
                    fn(stream)
                    stream.synchronize()
                except Exception as e:  # noqa: BLE001
                    # a host-side refusal is reported; a broken context ends the run
                    check_context(torch, tw, name)
                    kinds[name] = {"error": f"{type(e).__name__}: {e}", "in_step": False, "share_est": 0.0}
                    continue
            c0 = tw.bitnet_launch_count()
            try:
                g = capture(torch, stream, fn)
                kern = tw.bitnet_launch_count() - c0
                ms = time_graph(torch, stream, g, 3) / n_ops
            except Exception as e:  # noqa: BLE001
                if in_step:
                    raise
                check_context(torch, tw, name)
                kinds[name] = {"error": f"{type(e).__name__}: {e}", "in_step": False, "share_est": 0.0}
                continue
            reps_step = per_step * (a.decode_steps if name.startswith("decode") else 1)
            rate = work / (ms / 1e3) / (1e12 if bound == "tensor" else 1e9)
            peak = int8_peak_burst if bound == "tensor" else hbm_peak
            kinds[name] = {"us_per_op": ms * 1e3, "kernels_per_op": kern / n_ops, "bound": bound,
                           "work_per_op": work, "rate": rate, "rate_unit": "TOPS" if bound == "tensor" else "GB/s",
                           "frac_peak": rate / peak, "in_step": in_step,
                           "ops_per_step": reps_step if in_step else 0,
                           "share_est": ms * reps_step / ms_step if in_step else 0.0}
            del g
    dom = max(kinds, key=lambda k: kinds[k]["share_est"])
    d = kinds[dom]
    if d["bound"] == "hbm":
        achieved = d["work_per_op"] / (d["us_per_op"] / 1e6) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                "frac": achieved / hbm_peak}
    else:
        achieved = d["work_per_op"] / (d["us_per_op"] / 1e6) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": int8_peak_burst, "unit": "TFLOP/s",
                "frac": achieved / int8_peak_burst}
    roof["traffic"] = dram_traffic(dom)
    roof["kernel"] = dom
    roof["peak_source"] = f"{peaks_src} (MEASURED_PEAKS.json)" if peaks_src == "measured" else "fallback"
    if dom == "decode_sequence":
        roof["note"] = ("achieved = algorithmic bytes of one decode step (all packed weights of the stack + "
                        "activations in + outputs) / mean duration of one sequence launch in a CUDA graph of "
                        "consecutive decode steps (CUDA events on the launch stream)")
    else:
        roof["note"] = ("achieved = algorithmic bytes (packed weights + activations in + outputs) per op / "
                        "mean op time in a CUDA graph of consecutive ops (CUDA events on the launch stream)")

    # ---- configs 2 and 3: single BitLinears and FFNs at decode sizes ----
    configs = None
    if not a.no_configs:
        try:
            l2 = torch.cuda.get_device_properties(dev).L2_cache_size
            configs = decode_configs(st, stream, hbm_peak, l2)
        except Exception as e:  # noqa: BLE001
            check_context(torch, tw, "decode configs")
            configs = {"error": f"{type(e).__name__}: {e}"}

    # ---- end to end: pinned host inputs -> device, step, outputs -> host ----
    # Every step copies all of its inputs in from pinned host memory and all of the last layer's results
    # out.  The copies run on a second stream, ordered by events: step i + 1's prefill inputs go in, and
    # step i's prefill results come out, while step i's decode phase runs (the prefill inputs are dead
    # after the prefill pass; the prefill results are final after it).  The decode inputs go in and the
    # decode results come out around the decode phase.  The timed region spans all copies of all steps.
    e2e = None
    if a.e2e_steps > 0:
        h_pre = [x.cpu().pin_memory() for x in st.pre_x]
        h_dec = [x.cpu().pin_memory() for x in st.dec_x]
        outs_pre = list(st.pre_out.values())
        outs_dec = list(st.dec_out_l[-1].values())  # the last layer's decode results
        h_out_pre = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in outs_pre]
        h_out_dec = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in outs_dec]
        h2d = sum(x.numel() * x.element_size() for x in h_pre + h_dec)
        d2h = sum(o.numel() * o.element_size() for o in outs_pre + outs_dec)
        copy_stream = torch.cuda.Stream()

        def e2e_run(prefill, decode):
            ev = lambda: torch.cuda.Event()  # noqa: E731
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

            def copy_in(dst, src):
                for d_, h_ in zip(dst, src):
                    d_.copy_(h_, non_blocking=True)
                e = ev()
                e.record(copy_stream)
                return e

            def copy_out(dst, src):
                for h_, d_ in zip(dst, src):
                    h_.copy_(d_, non_blocking=True)
                e = ev()
                e.record(copy_stream)
                return e

            e0.record(stream)
            copy_stream.wait_event(e0)
            with torch.cuda.stream(copy_stream):
                pre_in, dec_in = copy_in(st.pre_x, h_pre), copy_in(st.dec_x, h_dec)
            pre_read = dec_read = None
            for i in range(a.e2e_steps):
                last = i + 1 == a.e2e_steps
                stream.wait_event(pre_in)
                if pre_read is not None:
                    stream.wait_event(pre_read)  # the previous step's prefill results are out
                prefill(stream)
                pre_free = ev()
                pre_free.record(stream)
                with torch.cuda.stream(copy_stream):
                    # while this step's decode phase runs: its prefill results out, the next step's prefill
                    # inputs in
                    copy_stream.wait_event(pre_free)
                    pre_read = copy_out(h_out_pre, outs_pre)
                    if not last:
                        pre_in = copy_in(st.pre_x, h_pre)
                stream.wait_event(dec_in)
                if dec_read is not None:
                    stream.wait_event(dec_read)
                decode(stream)
                dec_free = ev()
                dec_free.record(stream)
                with torch.cuda.stream(copy_stream):
                    copy_stream.wait_event(dec_free)
                    dec_read = copy_out(h_out_dec, outs_dec)
                    if not last:
                        dec_in = copy_in(st.dec_x, h_dec)
            stream.wait_event(pre_read)
            stream.wait_event(dec_read)
            e1.record(stream)
            e1.synchronize()
            return max_over_ranks(e0.elapsed_time(e1)) / a.e2e_steps

        def graphs_pre(s):
            g_pre.replay()

        def graphs_dec(s):
            for g in g_dec:
                g.replay()

        def eager_dec(s):
            for t in range(a.decode_steps):
                st.decode_step(t, s)

        torch.cuda.synchronize()
        barrier()
        with torch.cuda.stream(stream):
            e2e_ms = e2e_run(graphs_pre, graphs_dec)
        e2e = {"value": aggregate_value(n_gpus, tokens_step, Lyr, e2e_ms), "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
               "launch": "CUDA graphs of the step's calls; copies on a second stream, overlapping the decode phase"}
        # the same, with every projection called eagerly through the C ABI (argument checks, plan-cache
        # lookups and launches on the host, no graphs): what a caller without graphs gets
        torch.cuda.synchronize()
        barrier()
        t_host = time.perf_counter()
        with torch.cuda.stream(stream):
            eager_ms = e2e_run(st.prefill_pass, eager_dec)
        host_ms = (time.perf_counter() - t_host) * 1e3 / a.e2e_steps
        e2e["eager"] = {"value": aggregate_value(n_gpus, tokens_step, Lyr, eager_ms), "ms_per_step": eager_ms,
                        "host_ms_per_step": host_ms,
                        "calls_per_step": Lyr * 4 + (a.decode_steps if seq else a.decode_steps * Lyr * 4)}

    cpu = None
    if rank == 0 and n_gpus == 1 and not a.no_cpu_baseline:
        cpu = cpu_baseline(a.cpu_seconds)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": n_gpus, "steps": a.steps,
            "warmup": a.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int8", "data": "synthetic (seeded random activations and latents)",
            "config": workload_config(a, n_gpus), "phases": phases, "roofline": roof, "kernels": kinds,
            "decode_configs": configs,
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": int((launches_pre + launches_dec) * a.steps),
            "gpu_launches_per_step": {"prefill": int(launches_pre), "decode": int(launches_dec)},
            "clocks": clk, "gpu": torch.cuda.get_device_name(dev),
        }
        print(json.dumps(line), flush=True)
    del g_pre, g_dec
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    a = parse_args()
    n_gpus = int(os.environ.get("WORLD_SIZE", str(a.gpus)))
    if a.impl == "reference":
        return reference_arm(a, n_gpus)
    return our_arm(a, n_gpus)


if __name__ == "__main__":
    sys.exit(main())
