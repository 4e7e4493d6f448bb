"""Benchmark: compressed-KV decode attention on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload 0..4] [--layers L] [--context T] [--t-cap T]
                    [--quant 8|4] [--aware] [--seed S] [--no-cpu-baseline] [--no-clocks]

The default workload is the largest one-GPU configuration: LLaMA-7B attention
geometry (32 layers x 32 kv heads, MHA), 131072 tokens of context, ranks 48/64.

A step is one decode step of the whole model: for each of the workload's
layers, append the step's new token (projection, error, routing) and attend
over the layer's compressed cache with it included (append-then-attend), in
one lrkv_append_decode_attn call.  The same step as two calls
(lrkv_compress, then lrkv_decode_attn) is timed too and reported beside it.
Caches are built first by a prefill lrkv_compress per layer, which is timed
on its own (compress tokens/s).

Printed JSON line (rank 0):
  value   = decode-step algorithmic HBM bytes (all ranks) / max-over-ranks time, GB/s
  e2e     = the same through host buffers: pinned-host -> device copy of
            the step's inputs and device -> host copy of its outputs inside
            the timed region
  roofline: the decode kernel (with the fused append), the step's only launch
            per layer: algorithmic bytes per launch / its in-step duration (step
            time / layers), vs the measured copy bandwidth; the duration of each
            launch timed alone (events around it) is reported beside it as an
            upper bound on the time
  cpu_baseline: the fp64 CPU oracle on a bounded sample of the same work.

Multi-GPU (torchrun): every rank runs its own independent sequences (weak
scaling); no collective touches the data path, one all-reduce(max) gathers
the step time.
"""
import argparse
from dataclasses import replace
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402
from decode_attention_lrkv_b200 import accounting as A  # noqa: E402

HBM_SPEC_GBS = 8000.0
FALLBACK_PEAK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
FUSED_LAUNCHES = 1        # kernels one lrkv_append_decode_attn call launches
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", type=int, default=4)
    ap.add_argument("--t-cap", type=int, default=0,
                    help="cache capacity in positions (default: the context plus the appended steps)")
    ap.add_argument("--layers", type=int, default=0, help="override the layer count (testing)")
    ap.add_argument("--context", type=int, default=0,
                    help="override the context length (small profiling cases)")
    ap.add_argument("--quant", type=int, default=0, choices=[0, 8, 4],
                    help="stored coefficients as 8- or 4-bit codes with per-row scales (0: bf16)")
    ap.add_argument("--aware", action="store_true",
                    help="attention-aware key basis (query-side basis and key mean) in every layer")
    ap.add_argument("--seed", type=int, default=1234)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    return ap.parse_args()


def workload_of(args):
    over = {}
    if args.layers:
        over["layers"] = args.layers
    if args.context:
        over["T"] = args.context
    return synth.workload(args.workload, **over)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAK, "fallback"


# the decode kernel's sources: the stored ncu traffic is of the kernel built from these
DECODE_SOURCES = ("decode_stream.cuh", "decode_params.cuh", "decode_launch.cuh", "decode_simple.cuh",
                  "lrkv_common.cuh", "ptx.cuh", "launch_util.cuh")

# full-rank list capacity as a fraction of the cache capacity: the measured routed
# fraction is ~7-11% except on the 32K workload (r_k = 48 below the signal rank: 81%)
F_CAP_FRAC = {2: 1.0}
F_CAP_FRAC_DEFAULT = 0.25


def source_hash():
    """Hash of the decode kernel's sources: ties stored ncu traffic to the kernel it was taken on."""
    h = hashlib.sha256()
    cs = os.path.join(ROOT, "decode_attention_lrkv_b200", "csrc")
    for f in DECODE_SOURCES:
        with open(os.path.join(cs, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def stored_traffic(kernel, workload_name):
    if not os.path.exists(TRAFFIC_FILE):
        return None
    with open(TRAFFIC_FILE) as f:
        d = json.load(f)
    e = d.get(f"{kernel}@{workload_name}")
    if not e or e.get("source_hash") != source_hash():
        return None
    return e.get("bytes_per_launch")


class Clocks:
    """nvidia-smi samples (every 20 ms) from before the warm-up to after the timed region.

    Reported: the samples whose timestamps fall inside the timed region; when the
    region is shorter than the sampling interval, the samples of warm-up plus timed
    region (the GPU runs the same step throughout), marked as such."""
    Q = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, dev, enabled=True):
        self.p = None
        self.t_start = self.t_end = None
        self.out = os.path.join("/tmp", f"lrkv_clocks_{os.getpid()}.csv")
        if not enabled:
            return
        try:
            self.f = open(self.out, "w")
            uuid = str(torch.cuda.get_device_properties(dev).uuid)
            sel = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.p = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                       "-i", sel, "-lms", "20"], stdout=self.f,
                                      stderr=subprocess.DEVNULL)
            time.sleep(0.3)   # let the sampler come up before the warm-up starts
        except OSError:
            self.p = None

    def mark_start(self):
        self.t_start = time.time()

    def mark_end(self):
        self.t_end = time.time()

    @staticmethod
    def _stamp(s):
        import datetime
        try:
            return datetime.datetime.strptime(s, "%Y/%m/%d %H:%M:%S.%f").timestamp()
        except ValueError:
            return None

    def stop(self):
        if self.p is None:
            return None
        time.sleep(0.05)
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.p.kill()
        self.f.close()
        rows = []
        with open(self.out) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append((self._stamp(parts[0]), parts))
        os.unlink(self.out)
        window = "timed"
        sel = [r for ts, r in rows if ts is not None and self.t_start is not None
               and self.t_start <= ts <= self.t_end]
        if not sel:
            window = "warmup+timed"
            sel = [r for ts, r in rows if ts is not None and self.t_start is not None
                   and ts <= self.t_end and ts >= self.t_start - 2.0]
        if not sel:
            return None
        sm = [float(r[1]) for r in sel if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in sel if r[2].replace(".", "").isdigit()]
        reasons = sorted({self.NAMES[i] for r in sel for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(sel),
                "window": window}


# ---------------------------------------------------------------------------
# ranks: one process per GPU; each runs its own independent sequences
# ---------------------------------------------------------------------------

def rank_seed(seed, rank):
    """Seed of a rank's synthetic inputs: every rank draws different sequences."""
    return seed + 7919 * rank


def max_over_ranks(x, dev, world):
    """The largest value over the ranks (the slowest rank's time); every rank calls it."""
    if world <= 1:
        return float(x)
    t = torch.tensor([float(x)], device=dev, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x, dev, world):
    """The sum over the ranks (the whole job's bytes); every rank calls it."""
    if world <= 1:
        return float(x)
    t = torch.tensor([float(x)], device=dev, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return float(t.item())


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def aware_key_basis(U_k, seed, layer):
    """An attention-aware key basis of Theorem 1's form (NOVA-KV summary) for a
    query covariance whose eigenvectors are U_k's columns: the key-side basis
    W_k = U_k diag(s), the query-side basis W_q = U_k diag(1/s), s the square
    roots of seeded query-covariance eigenvalues, and a seeded key mean inside
    span(U_k).  Then W_q W_k^T = U_k U_k^T (up to bf16 rounding) and the mean
    lies in the span, so the routed set is that of the plain basis and the step
    moves the same bytes: what the timing shows is the cost of the query-side
    basis and the mean in the kernels."""
    g = torch.Generator(device=U_k.device).manual_seed(int(seed) * 7919 + int(layer))
    Hkv, d, r = U_k.shape
    s = torch.exp(0.5 * torch.randn(Hkv, 1, r, generator=g, device=U_k.device))
    W_k = (U_k.float() * s).to(torch.bfloat16)
    W_q = (U_k.float() / s).to(torch.bfloat16)
    m = 0.05 * torch.randn(Hkv, r, 1, generator=g, device=U_k.device)
    mu = torch.matmul(U_k.float(), m).squeeze(-1)
    return W_k, W_q, mu


def build_layers(L, w, seed, steps_total, dev, workload_id, t_cap=0, aware=False, quant=0):
    """Prefill every layer's cache through lrkv_compress; time each prefill.

    Each timed prefill starts with a cold L2 (a 256 MB buffer is written first)
    and behind a short device-side sleep, so that the host-side launch work of
    the call overlaps the sleep and the events bracket device time only.  One
    untimed prefill into a scratch cache first loads the kernels."""
    T_cap = synth.pad_to(max(w.T + steps_total + 1, t_cap), 32)
    F_cap = synth.pad_to(int(F_CAP_FRAC.get(workload_id, F_CAP_FRAC_DEFAULT) * T_cap), 32)
    dims = L.Dims(B=w.B, Hq=w.Hq, Hkv=w.Hkv, d=w.d, r_k=w.r_k, r_v=w.r_v, T_cap=T_cap, F_cap=F_cap,
                  coef_bits=quant)
    ws = L.make_workspace(dims, dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    layers = []
    comp_ms = []
    lengths = None
    for li in range(w.layers):
        lay = synth.make_layer(w, li, seed, device=dev)
        lengths = lay["lengths"]
        t_new_b = (lengths.to(torch.int32).to(dev) if w.ragged_min else None)
        kb = {}
        if aware:
            W_k, W_q, mu = aware_key_basis(lay["U_k"], seed, li)
            kb = dict(U_kq=W_q, mu_k=mu)
            lay["U_k"] = W_k
        if li == 0:
            scratch = L.LayerCache(dims, lay["U_k"], lay["U_v"], device=dev, **kb)
            L.lrkv_compress(dims, scratch, lay["K"], lay["V"], w.tau, t_new_b=t_new_b, ws=ws)
            torch.cuda.synchronize()
            del scratch
        cache = L.LayerCache(dims, lay["U_k"], lay["U_v"], device=dev, **kb)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        flush.zero_()
        torch.cuda._sleep(1_000_000)
        e0.record()
        L.lrkv_compress(dims, cache, lay["K"], lay["V"], w.tau, t_new_b=t_new_b, ws=ws)
        e1.record()
        torch.cuda.synchronize()
        comp_ms.append(e0.elapsed_time(e1))
        Ka, Va = synth.decode_tokens(w, lay["Qk"], lay["Qv"], steps_total, seed, li, dev)
        qa = synth.decode_queries(w, steps_total, seed, li, dev)
        layers.append(dict(cache=cache, K_app=Ka, V_app=Va, q_app=qa))
        del lay
    del flush
    return dims, ws, layers, comp_ms, lengths


def capture_step_graph(L, dims, ws, layers, w, s, out, dec_events, host=None, fused=True):
    """One CUDA graph: every layer's append + decode for step s.

    fused: one lrkv_append_decode_attn call per layer, else lrkv_compress then
    lrkv_decode_attn.  host: optional (pinned inputs, pinned outputs, device
    staging) for the end-to-end variant with copies in the graph.
    """
    g = torch.cuda.CUDAGraph()
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        with torch.cuda.graph(g, stream=stream):
            if host is not None:   # the step's inputs for every layer: one copy per tensor
                hin, hout, stage = host
                for name in ("k", "v", "q"):
                    stage[name].copy_(hin[name][s], non_blocking=True)
            for li, lay in enumerate(layers):
                if host is not None:
                    k, v, q = stage["k"][li], stage["v"][li], stage["q"][li]
                else:
                    k = lay["K_app"][:, s:s + 1]
                    v = lay["V_app"][:, s:s + 1]
                    q = lay["q_app"][s]
                if not fused:
                    L.lrkv_compress(dims, lay["cache"], k, v, w.tau, ws=ws, stream=stream)
                if dec_events is not None:
                    dec_events[li][0].record(stream)
                if fused:
                    L.lrkv_append_decode_attn(dims, lay["cache"], k, v, w.tau, q, out[li], ws=ws,
                                              stream=stream)
                else:
                    L.lrkv_decode_attn(dims, lay["cache"], q, out[li], ws=ws, stream=stream)
                if dec_events is not None:
                    dec_events[li][1].record(stream)
            if host is not None:   # the step's result for every layer: one copy back
                hout[s].copy_(out, non_blocking=True)
    torch.cuda.current_stream().wait_stream(stream)
    return g


def run_ours(args, rank, world, dev):
    import decode_attention_lrkv_b200 as L
    L.load_library()
    w = workload_of(args)
    K, W = args.steps, args.warmup
    steps_total = W + K
    seed = rank_seed(args.seed, rank)
    dims, ws, layers, comp_ms, lengths = build_layers(L, w, seed, 4 * steps_total, dev, args.workload,
                                                      args.t_cap, aware=args.aware, quant=args.quant)
    out = torch.empty(w.layers, w.B, w.Hq, w.d, dtype=torch.float32, device=dev)

    # --- device-resident timed region: the step graphs carry no events (an event
    # node between two kernels costs microseconds and stops the dependent launch
    # overlap), so the step time is the kernels' own ---------------------------------
    graphs = [capture_step_graph(L, dims, ws, layers, w, s, out, None) for s in range(steps_total)]
    torch.cuda.synchronize()
    clocks = Clocks(dev, enabled=not args.no_clocks)
    for s in range(W):
        graphs[s].replay()
    torch.cuda.synchronize()
    seq_before = layers[0]["cache"].seq_len.cpu().tolist()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks.mark_start()
    t0.record()
    for s in range(W, steps_total):
        graphs[s].replay()
    t1.record()
    torch.cuda.synchronize()
    clocks.mark_end()
    if world > 1:
        torch.distributed.barrier()
    clk = clocks.stop()
    ms = t0.elapsed_time(t1)
    for g in graphs:
        g.reset()
    del graphs
    full_cnt = [lay["cache"].full_cnt.cpu().numpy() for lay in layers]
    ms = max_over_ranks(ms, dev, world)

    # --- the decode kernel's own launch duration: the same steps again, with
    # CUDA events recorded on the launching stream around every decode ----------------
    ev = [[[torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)]
           for _ in range(w.layers)] for _ in range(steps_total)]
    graphs = [capture_step_graph(L, dims, ws, layers, w, s, out, ev[s]) for s in range(steps_total)]
    torch.cuda.synchronize()
    for s in range(W):
        graphs[s].replay()
    torch.cuda.synchronize()
    seq_k = layers[0]["cache"].seq_len.cpu().tolist()
    for s in range(W, steps_total):
        graphs[s].replay()
    torch.cuda.synchronize()
    full_cnt_k = [lay["cache"].full_cnt.cpu().numpy() for lay in layers]
    dec_ms = [ev[s][li][0].elapsed_time(ev[s][li][1]) for s in range(W, steps_total)
              for li in range(w.layers)]
    for g in graphs:
        g.reset()
    del graphs

    # --- the same step as two calls per layer (lrkv_compress, lrkv_decode_attn) ---------
    graphs = [capture_step_graph(L, dims, ws, layers, w, s, out, None, fused=False)
              for s in range(steps_total)]
    torch.cuda.synchronize()
    for s in range(W):
        graphs[s].replay()
    torch.cuda.synchronize()
    u0, u1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    u0.record()
    for s in range(W, steps_total):
        graphs[s].replay()
    u1.record()
    torch.cuda.synchronize()
    unfused_ms = max_over_ranks(u0.elapsed_time(u1), dev, world) / K
    for g in graphs:
        g.reset()
    del graphs

    # --- the decode kernel back to back: one graph of every layer's decode, K times
    # (no appends: the caches stay as they are), so consecutive decodes overlap as
    # they do behind an append -------------------------------------------------------
    chain_graph = torch.cuda.CUDAGraph()
    cstream = torch.cuda.Stream()
    cstream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cstream):
        for li, lay in enumerate(layers):   # load outside the capture
            L.lrkv_decode_attn(dims, lay["cache"], lay["q_app"][0], out[li], ws=ws, stream=cstream)
        with torch.cuda.graph(chain_graph, stream=cstream):
            for _ in range(K):
                for li, lay in enumerate(layers):
                    L.lrkv_decode_attn(dims, lay["cache"], lay["q_app"][0], out[li], ws=ws,
                                       stream=cstream)
    torch.cuda.current_stream().wait_stream(cstream)
    torch.cuda.synchronize()
    chain_graph.replay()
    torch.cuda.synchronize()
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    c0.record()
    chain_graph.replay()
    c1.record()
    torch.cuda.synchronize()
    chain_launch_ms = c0.elapsed_time(c1) / (K * w.layers)
    chain_graph.reset()
    del chain_graph
    seq_c = layers[0]["cache"].seq_len.cpu().tolist()
    full_cnt_c = [lay["cache"].full_cnt.cpu().numpy() for lay in layers]

    # algorithmic bytes of the timed steps: step s attends over seq_len + 1 tokens
    T_mid = [int(x) + (K + 1) / 2.0 for x in seq_before]
    dec_bytes = [A.decode_bytes(w.B, w.Hq, w.Hkv, w.d, w.r_k, w.r_v, T_mid, fc, coef_bits=dims.bits) for fc in full_cnt]
    routed_frac = float(sum(fc.sum() for fc in full_cnt)) / (w.layers * w.Hkv * sum(T_mid))
    app_bytes = A.compress_bytes(w.Hkv, w.d, w.r_k, w.r_v, w.B, w.B * w.Hkv * routed_frac,
                                 coef_bits=dims.bits)
    step_bytes = sum(dec_bytes) + w.layers * app_bytes
    ms_step = ms / K
    value = sum_over_ranks(step_bytes, dev, world) / (ms_step * 1e-3) / 1e9
    dec_launch_ms = float(np.mean(dec_ms))
    T_mid_k = [int(x) + (K + 1) / 2.0 for x in seq_k]
    dec_bytes_launch = float(np.mean([A.decode_bytes(w.B, w.Hq, w.Hkv, w.d, w.r_k, w.r_v, T_mid_k, fc, coef_bits=dims.bits)
                                      for fc in full_cnt_k])) + app_bytes   # the fused append's too
    pk, pk_kind = peaks()
    peak = pk.get("hbm_gbs", FALLBACK_PEAK["hbm_gbs"])
    # in-step: the fused call is the step's only launch per layer, so a layer's
    # share of the step time is that launch's duration inside the step
    layer_ms = ms_step / w.layers
    layer_bytes = step_bytes / w.layers
    achieved = layer_bytes / (layer_ms * 1e-3) / 1e9
    isolated = dec_bytes_launch / (dec_launch_ms * 1e-3) / 1e9
    dec_bytes_chain = float(np.mean([A.decode_bytes(w.B, w.Hq, w.Hkv, w.d, w.r_k, w.r_v,
                                                    [int(x) for x in seq_c], fc, coef_bits=dims.bits) for fc in full_cnt_c]))
    chained = dec_bytes_chain / (chain_launch_ms * 1e-3) / 1e9
    status = max(int(lay["cache"].dev_status[0].item()) for lay in layers)

    # --- prefill compress rate ----------------------------------------------------------
    n_tok = float(sum(int(x) for x in lengths))
    comp_tok_s = n_tok / (float(np.mean(comp_ms)) * 1e-3)
    comp_bytes = A.compress_bytes(w.Hkv, w.d, w.r_k, w.r_v, n_tok, n_tok * w.Hkv * routed_frac,
                                  coef_bits=dims.bits)
    comp_tflops = A.compress_tc_flops(w.Hkv, w.d, w.r_k, w.r_v, n_tok) / (float(np.mean(comp_ms)) * 1e-3) / 1e12

    # --- end-to-end through host buffers --------------------------------------------------
    e2e = run_e2e(L, args, w, dims, ws, layers, dev, world, steps_total)
    side = side_measurements(L, w, dims, layers, dev, pk)

    result = {
        "metric": "compressed-KV decode attn µs/step & HBM GB/s vs 8 TB/s; compress tok/s",
        "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": round(ms_step, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "layers": w.layers, "batch": w.B, "context": w.T,
                   "T_cap": dims.T_cap, "F_cap": dims.F_cap,
                   "key_basis": ("attention-aware (query-side basis + key mean)" if args.aware
                                 else "orthonormal (StaticPCA)"),
                   "coefficients": "bf16" if dims.bits == 16 else f"int{dims.bits} codes + fp32 row scales",
                   "bytes_per_compressed_token_head": A.compressed_bytes_per_token_head(
                       w.r_k, w.r_v, coef_bits=dims.bits),
                   "q_heads": w.Hq, "kv_heads": w.Hkv, "head_dim": w.d, "r_k": w.r_k, "r_v": w.r_v,
                   "tau": w.tau, "parallelism": f"replicas{world}" if world > 1 else "single",
                   "l2": f"inputs larger than L2: {step_bytes / 1e9:.2f} GB touched per step vs 126 MB L2",
                   "graph": "one CUDA graph per step (all layers: fused append + decode)"},
        "us_per_step": round(ms_step * 1e3, 2),
        "frac_of_8TBs": round(value / world / HBM_SPEC_GBS, 4),
        "routed_fraction": round(routed_frac, 4),
        "dev_status": status,
        "compress": {"tok_per_s_per_layer": round(comp_tok_s, 1),
                     "us_per_layer": round(float(np.mean(comp_ms)) * 1e3, 2),
                     "gbs": round(comp_bytes / (float(np.mean(comp_ms)) * 1e-3) / 1e9, 2),
                     "frac_of_measured_hbm": round(comp_bytes / (float(np.mean(comp_ms)) * 1e-3) / 1e9
                                                   / pk.get("hbm_gbs", FALLBACK_PEAK["hbm_gbs"]), 4),
                     "tensor_tflops_executed": round(comp_tflops, 1),
                     "tensor_frac_of_measured_bf16": round(comp_tflops / pk.get("bf16_tflops",
                                                                                FALLBACK_PEAK["bf16_tflops"]), 4),
                     "tokens_per_layer": n_tok},
        "unfused_step": {"us_per_step": round(unfused_ms * 1e3, 2),
                         "value": round(sum_over_ranks(step_bytes, dev, world) / (unfused_ms * 1e-3) / 1e9, 2),
                         "calls": "lrkv_compress then lrkv_decode_attn per layer (two launches)"},
        "roofline": {"kernel": "decode_stream_kernel (fused append + decode)", "bound": "hbm",
                     "achieved": round(achieved, 2), "peak": peak,
                     "peak_kind": pk_kind + " copy bandwidth", "unit": "GB/s",
                     "frac": round(achieved / peak, 4),
                     "frac_of_8TBs": round(achieved / HBM_SPEC_GBS, 4),
                     "traffic": stored_traffic("decode_attn", w.name),
                     "algorithmic_bytes_per_launch": round(layer_bytes),
                     "us_per_launch": round(layer_ms * 1e3, 3),
                     "launch_timing": "in-step: the timed step time / layers (one fused launch per "
                                      "layer and nothing else in the step), CUDA events around K "
                                      "replays of the step graphs",
                     "isolated_launch": {"us_per_launch": round(dec_launch_ms * 1e3, 3),
                                         "achieved": round(isolated, 2),
                                         "frac": round(isolated / peak, 4),
                                         "timing": "CUDA events on the launching stream around every "
                                                   "fused call, in a second pass of the same steps; "
                                                   "the events stop the dependent-launch overlap, so "
                                                   "this is an upper bound on the in-step time"},
                     "chained": {"us_per_launch": round(chain_launch_ms * 1e3, 3),
                                 "achieved": round(chained, 2),
                                 "frac": round(chained / peak, 4),
                                 "timing": "one CUDA graph of every layer's decode, K times back "
                                           "to back (no appends), CUDA events around the replay"}},
        "e2e": e2e,
        "side": side,
        "gpu_launches": K * w.layers * (FUSED_LAUNCHES if dims.bits != 4 and w.g in (1, 2, 4)
                                        else 2),   # 4-bit codes or other groups: append + decode
        "clocks": clk,
    }
    return result, w, layers, dims


def _event_time_ms(fn, reps, warm=3):
    """Mean device time of fn() over reps calls, CUDA events around the batch."""
    for _ in range(warm):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def side_measurements(L, w, dims, layers, dev, pk):
    """Timings of the calls the step does not use, on this workload's geometry:
    the online basis update (one Oja batch step of every kv head's key basis
    over 4096 rows) and the decode with other query groups on layer 0's cache
    (the cache does not depend on the query heads): GQA 3 (one launch of the
    streaming kernel, 4 heads with one idle) and GQA 8 (two launches of 4
    heads, each streaming the cache)."""
    out = {}
    g = torch.Generator(device=dev).manual_seed(99)
    n_rows = 4096
    X = torch.randn(n_rows, w.Hkv, w.d, generator=g, device=dev).to(torch.bfloat16)
    U = torch.linalg.qr(torch.randn(w.Hkv, w.d, w.r_k, generator=g, device=dev, dtype=torch.float64))[0].float()
    Ub = torch.empty(w.Hkv, w.d, w.r_k, dtype=torch.bfloat16, device=dev)
    ows = torch.empty(L.lrkv_oja_workspace_size(dims, n_rows, w.r_k), dtype=torch.uint8, device=dev)
    ms = _event_time_ms(lambda: L.lrkv_oja_update(dims, X, U, 1e-3, U_out=Ub, ws=ows), 10)
    flops = 4.0 * n_rows * w.d * w.r_k * w.Hkv
    out["oja_update"] = {"us_per_call": round(ms * 1e3, 2), "rows": n_rows, "kv_heads": w.Hkv,
                         "rank": w.r_k, "tflops": round(flops / (ms * 1e-3) / 1e12, 3),
                         "note": "one batch step (sums on CUDA cores in fp32, fp64 step + Gram-Schmidt)"}
    lay = layers[0]
    fb = {}
    for gg in (3, 8):
        Dg = L.Dims(B=dims.B, Hq=gg * dims.Hkv, Hkv=dims.Hkv, d=dims.d, r_k=dims.r_k, r_v=dims.r_v,
                    T_cap=dims.T_cap, F_cap=dims.F_cap, coef_bits=dims.coef_bits)
        wsg = L.make_workspace(Dg, dev)
        q = torch.randn(dims.B, Dg.Hq, dims.d, generator=g, device=dev).to(torch.bfloat16)
        o = torch.empty(dims.B, Dg.Hq, dims.d, dtype=torch.float32, device=dev)
        ms = _event_time_ms(lambda: L.lrkv_decode_attn(Dg, lay["cache"], q, o, ws=wsg), 10)
        fc = lay["cache"].full_cnt.cpu().numpy()
        nb = A.decode_bytes(Dg.B, Dg.Hq, Dg.Hkv, Dg.d, Dg.r_k, Dg.r_v, lay["cache"].seq_len.cpu().tolist(), fc,
                            coef_bits=dims.bits)
        fb[f"gqa{gg}"] = {"us_per_call": round(ms * 1e3, 2), "gbs": round(nb / (ms * 1e-3) / 1e9, 1),
                          "frac_of_measured_hbm": round(nb / (ms * 1e-3) / 1e9 / pk.get("hbm_gbs", 6549.1), 4)}
        del wsg
    out["gqa_decode"] = fb
    return out


def run_e2e(L, args, w, dims, ws, layers, dev, world, steps_total):
    """The step again, inputs from pinned host memory and outputs back to it."""
    K, W = args.steps, args.warmup
    n = steps_total
    hin = {"k": torch.empty(n, w.layers, w.B, 1, w.Hkv, w.d, dtype=torch.bfloat16).pin_memory(),
           "v": torch.empty(n, w.layers, w.B, 1, w.Hkv, w.d, dtype=torch.bfloat16).pin_memory(),
           "q": torch.empty(n, w.layers, w.B, w.Hq, w.d, dtype=torch.bfloat16).pin_memory()}
    for li, lay in enumerate(layers):
        hin["k"][:, li].copy_(lay["K_app"][:, 2 * steps_total:3 * steps_total].permute(1, 0, 2, 3).unsqueeze(2).cpu())
        hin["v"][:, li].copy_(lay["V_app"][:, 2 * steps_total:3 * steps_total].permute(1, 0, 2, 3).unsqueeze(2).cpu())
        hin["q"][:, li].copy_(lay["q_app"][2 * steps_total:3 * steps_total].cpu())
    hout = torch.empty(n, w.layers, w.B, w.Hq, w.d, dtype=torch.float32).pin_memory()
    stage = {"k": torch.empty(w.layers, w.B, 1, w.Hkv, w.d, dtype=torch.bfloat16, device=dev),
             "v": torch.empty(w.layers, w.B, 1, w.Hkv, w.d, dtype=torch.bfloat16, device=dev),
             "q": torch.empty(w.layers, w.B, w.Hq, w.d, dtype=torch.bfloat16, device=dev)}
    out = torch.empty(w.layers, w.B, w.Hq, w.d, dtype=torch.float32, device=dev)
    graphs = [capture_step_graph(L, dims, ws, layers, w, s, out, None, host=(hin, hout, stage))
              for s in range(n)]
    torch.cuda.synchronize()
    for s in range(W):
        graphs[s].replay()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for s in range(W, n):
        graphs[s].replay()
    t1.record()
    torch.cuda.synchronize()
    ms = max_over_ranks(t0.elapsed_time(t1), dev, world)
    for g in graphs:
        g.reset()
    T_now = [int(x) for x in layers[0]["cache"].seq_len.cpu()]
    T_mid = [t - (K - 1) / 2.0 for t in T_now]
    full_cnt = [lay["cache"].full_cnt.cpu().numpy() for lay in layers]
    step_bytes = sum(A.decode_bytes(w.B, w.Hq, w.Hkv, w.d, w.r_k, w.r_v, T_mid, fc, coef_bits=dims.bits) for fc in full_cnt)
    step_bytes += w.layers * A.compress_bytes(w.Hkv, w.d, w.r_k, w.r_v, w.B, 0, coef_bits=dims.bits)
    h2d = sum(t[0].numel() * t[0].element_size() for t in hin.values())
    d2h = hout[0].numel() * hout[0].element_size()
    job_bytes = sum_over_ranks(step_bytes, dev, world)
    return {"value": round(job_bytes / (ms / K * 1e-3) / 1e9, 2), "unit": "GB/s",
            "us_per_step": round(ms / K * 1e3, 2), "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h)}


# ---------------------------------------------------------------------------
# the fp64 CPU oracle: baseline leg of our arm, and the reference arm
# ---------------------------------------------------------------------------

def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


ORACLE_MAX_TOKEN_HEADS = 1 << 18


def oracle_sample_workload(w):
    """The bounded sample of workload w that the oracle runs: the same sizes,
    ranks and input recipe with fewer kv heads (and their query heads) when
    B * T * Hkv exceeds ORACLE_MAX_TOKEN_HEADS, so one oracle step stays well
    under a second."""
    h = max(1, min(w.Hkv, ORACLE_MAX_TOKEN_HEADS // (w.B * w.T)))
    return replace(w, Hkv=h, Hq=h * w.g)


class OracleLayer:
    """One layer of the workload in the fp64 oracle: prefill once, then decode steps."""

    def __init__(self, w, li, seed, n_steps):
        import oracle as O
        self.O, self.w = O, w
        lay = synth.make_layer(w, li, seed, device="cpu")
        f64 = lambda t: t.double().numpy()
        T_cap = synth.pad_to(w.T + n_steps + 1, 32)
        D = O.Dims(B=w.B, Hq=w.Hq, Hkv=w.Hkv, d=w.d, r_k=w.r_k, r_v=w.r_v, T_cap=T_cap, F_cap=T_cap)
        self.c = O.Cache.empty(D, f64(lay["U_k"]), f64(lay["U_v"]))
        lengths = lay["lengths"].tolist()
        t = time.perf_counter()
        O.compress(self.c, f64(lay["K"]), f64(lay["V"]), w.tau,
                   t_new_b=lengths if w.ragged_min else None)
        self.prefill_s = time.perf_counter() - t
        self.prefill_tokens = sum(lengths)
        Ka, Va = synth.decode_tokens(w, lay["Qk"], lay["Qv"], n_steps, seed, li, "cpu")
        self.K, self.V = f64(Ka), f64(Va)
        self.q = f64(synth.decode_queries(w, n_steps, seed, li, "cpu"))
        self.s = 0

    def step(self):
        """One timed decode step of this layer: append the step's token, then attend."""
        O, w, s = self.O, self.w, self.s
        t = time.perf_counter()
        O.compress(self.c, self.K[:, s:s + 1], self.V[:, s:s + 1], w.tau)
        O.decode_attn(self.c, self.q[s])
        dt = time.perf_counter() - t
        self.s += 1
        nbytes = A.decode_bytes(w.B, w.Hq, w.Hkv, w.d, w.r_k, w.r_v, self.c.seq_len.tolist(),
                                self.c.full_cnt) + A.compress_bytes(w.Hkv, w.d, w.r_k, w.r_v, w.B, 0)
        return nbytes, dt


def oracle_sample(w, seed, timed_budget_s=12.0, max_steps=600):
    """The oracle on decode steps of layer 0 of the workload until ~timed_budget_s.

    Setup (the layer's prefill through the oracle) is untimed but its tokens/s
    is reported.  Returns (GB/s of algorithmic decode-step bytes, compress
    tokens/s, steps, timed s).
    """
    ol = OracleLayer(oracle_sample_workload(w), 0, seed, max_steps)
    nbytes = secs = 0.0
    n = 0
    while n < max_steps and secs < timed_budget_s:
        b, dt = ol.step()
        nbytes, secs = nbytes + b, secs + dt
        n += 1
    return nbytes / secs / 1e9, ol.prefill_tokens / ol.prefill_s, n, secs


def run_reference(args):
    w = workload_of(args)
    ws = oracle_sample_workload(w)
    # setup (untimed): the oracle prefills one layer (of ws.Hkv kv heads); each step
    # is one oracle decode step over that layer -- a bounded sample of the workload's step
    ol = OracleLayer(ws, 0, args.seed, args.warmup + args.steps)
    for _ in range(args.warmup):
        ol.step()
    nbytes = secs = 0.0
    for _ in range(args.steps):
        b, dt = ol.step()
        nbytes, secs = nbytes + b, secs + dt
    value = nbytes / secs / 1e9
    cores = blas_threads()
    sample = (f"one of {w.layers} layers of {w.name} per step, {ws.Hkv} of its {w.Hkv} kv heads "
              f"(B={w.B}, T={w.T}): fp64 oracle append + decode, {args.steps} steps, {secs:.2f} s timed")
    return {"impl": "reference",
            "metric": "compressed-KV decode attn µs/step & HBM GB/s vs 8 TB/s; compress tok/s",
            "value": round(value, 4), "unit": "GB/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(secs / args.steps * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": w.name, "layers_per_step": 1},
            "compress": {"tok_per_s_per_layer": round(ol.prefill_tokens / ol.prefill_s, 1)},
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return 0
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the library has no CPU path)")
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=dev)
    result, w, layers, dims = run_ours(args, rank, world, dev)
    if rank == 0 and not args.no_cpu_baseline:
        v, ctok, n, secs = oracle_sample(w, args.seed)
        hs = oracle_sample_workload(w).Hkv
        result["cpu_baseline"] = {
            "value": round(v, 4), "unit": "GB/s", "cores": blas_threads(), "kind": "oracle",
            "compress_tok_per_s_per_layer": round(ctok, 1),
            "sample": f"{n} decode steps (append + attend) of layer 0 of {w.name}, {hs} of its "
                      f"{w.Hkv} kv heads (1 of {w.layers} layers, B={w.B}, T={w.T}): fp64 oracle, "
                      f"{secs:.1f} s timed; the layer's prefill through the oracle timed separately "
                      f"(tokens/s over those heads)"}
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
