"""Decode-step benchmark of libspectra on B200.

One step = one decode step through a stack of attention layers shaped like the
named workload: per layer, spectra_encode_append of each sequence's new token
(projection + quantise + pack + append, one fused kernel) followed by
spectra_decode_attend over the whole latent cache (one kernel).  Caches and codec
factors of all layers (> L2) are resident in HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload stress|qwen|llama]
                    [--extra qwen,llama,prefill] [--check] [--impl ours|reference]
                    [--decode latent|reconstruct] [--rope-theta T]

Prints one JSON line (rank 0).  Its top-level figures are the --workload's
(default: the 12x heavy-tail stress layer, batch 16 at 32k context); the --extra
workloads' records (default: Qwen-shaped 8x at 128k, Llama-shaped 4x at 32k, and
the 65,536-token prefill encode) are nested under "workloads".  Metric: cache
tokens/s/head = sum over layers of batch * context * n_kv_heads per second of
step time.  ``roofline`` reports the decode kernel against the measured HBM copy
bandwidth over the packed bytes it must read.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

MODEL_LAYERS = {"llama": 32, "qwen": 28, "stress": 32}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]), "src": "measured"}
    return dict(FALLBACK_PEAKS, src="fallback")


def max_over_ranks(values, device):
    """Element-wise maximum of per-rank timings over the process group (the job
    takes as long as its slowest rank); NCCL needs device tensors, gloo host ones."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.cpu()]


def replicas_throughput(units_per_step_per_rank, ms_per_step_max, world):
    """Whole-job throughput of `world` independent replicas (weak scaling): the
    units all ranks processed per step over the slowest rank's step time."""
    return units_per_step_per_rank * world / (ms_per_step_max / 1e3)


def _workload_name(cfg, layers):
    return (f"{cfg.name}: {layers} layers x (d_model {cfg.d_model}, {cfg.n_q_heads}q/{cfg.n_kv_heads}kv heads, "
            f"d_head {cfg.d_head}, groups of {cfg.group}, {cfg.budget_bits} bits/side), "
            f"batch {cfg.batch} decode at {cfg.cache_len} context")


# ---------------------------------------------------------------------------
# CPU oracle baseline (bounded sample of the same workload)
# ---------------------------------------------------------------------------
# DRAM bytes (read + write) per algorithmic byte of one launch of a kernel, from
# one ncu capture of the current kernel on a 1-layer case of the workload; a
# workload/kernel without a capture of its current code reports traffic null.
#   attend_kernel, stress 12x (128-token pages), batch 16 x 32,771 tokens:
#     169,200,128 B read + 4,024,064 B written for 167,787,520 packed bytes
#   attend_kernel, Qwen 8x, 131,075 tokens: 34,037,504 B read, 0 written, for
#     33,555,200 packed bytes
#   rt_split_kernel (tiles staged by cp.async), Llama-shaped, 32k context:
#     34,244,608 B read, 0 written, for 33,560,576 packed bytes
TRAFFIC_PER_ALGO_BYTE = {"stress": (169_200_128 + 4_024_064) / 167_787_520, "qwen": 34_037_504 / 33_555_200}
TRAFFIC_PER_PACKED_BYTE_RT = {"llama": 34_244_608 / 33_560_576}


def _oracle_decode_case(cfg, n_tok=8192, rope_theta=None):
    """One KV head of the workload's layer for the CPU oracle: widths from the
    workload's spectrum, a packed pool of ``n_tok`` seeded tokens, W_up, queries.
    rope_theta None: the latent decode's reference; else reconstruct-then-attend
    with that rotary base."""
    import numpy as np

    import oracle

    rng = np.random.default_rng(cfg.seed)
    s2 = np.arange(1, cfg.rank + 1) ** -cfg.spectrum_exp
    widths = oracle.allocate_widths(s2, cfg.group, cfg.budget_bits, cfg.count_overhead)
    w1 = [[widths, widths]]
    P = cfg.page_tokens
    lay = oracle.page_layout(w1, cfg.group, P)
    pool = np.zeros(lay["page_bytes"] * (n_tok // P), np.uint8)
    table = np.arange(n_tok // P)[None, :]
    nk = int(sum(cfg.group for b in widths if b > 0))
    lat = (rng.standard_normal((n_tok, 2 * nk)) * 0.3).astype(np.float32)
    oracle.append_tokens(pool, lay["page_bytes"], lay, w1, cfg.group, P, table, np.zeros(1),
                         np.zeros(n_tok, np.int64), lat, 1)
    q, _ = np.linalg.qr(rng.standard_normal((cfg.d_head, cfg.d_head)))
    W_up = [[q[:nk].astype(np.float32), q[:nk].astype(np.float32)]]
    qs = rng.standard_normal((1, cfg.gq, cfg.d_head)).astype(np.float32)

    def run(tokens):
        if rope_theta is None:
            oracle.decode_reference(pool, lay["page_bytes"], lay, cfg.group, P, table, np.array([tokens]), qs,
                                    W_up, cfg.gq, 1)
        else:
            oracle.decode_reference_rope(pool, lay["page_bytes"], lay, cfg.group, P, table, np.array([tokens]), qs,
                                         W_up, cfg.gq, 1, rope_theta)
    return run, n_tok


def _blas_threads():
    # numpy runs the unpacking and softmax on one thread; only the BLAS matmuls
    # (rebuilding K and V from the latents) fan out, to the BLAS pool's threads
    try:
        from threadpoolctl import threadpool_info
        return max([d["num_threads"] for d in threadpool_info() if d.get("user_api") == "blas"] or [1])
    except Exception:
        return 1


def _sample_text(cfg, tokens, what):
    return (f"oracle decode of 1 KV head ({cfg.gq} q heads) over {tokens} of {cfg.cache_len} context tokens "
            f"of one {cfg.name} layer, {what}; numpy float64, unpacking on one thread, BLAS matmuls on "
            f"{_blas_threads()} threads of {os.cpu_count()} host cores")


def cpu_oracle_sample(cfg, target_s=12.0, rope_theta=None):
    """The oracle's decode throughput over a bounded sample (about ``target_s`` s)."""
    run, n_tok = _oracle_decode_case(cfg, rope_theta=rope_theta)
    t0 = time.perf_counter()
    reps = 0
    while True:
        run(n_tok)
        reps += 1
        el = time.perf_counter() - t0
        if el >= target_s:
            break
    value = reps * n_tok / el  # tokens/s/head (one KV head per pass)
    what = f"{reps} passes in {el:.1f} s"
    if rope_theta is not None:
        what += f", reconstruct-then-attend with rotary base {rope_theta:g}"
    return value, _blas_threads(), _sample_text(cfg, n_tok, what)


def cpu_oracle_steps(cfg, steps, warm, budget_s=120.0, rope_theta=None):
    """The oracle as the reference arm: ``warm`` untimed and ``steps`` timed steps,
    each the decode of one KV head over a context sample sized so that the whole
    run takes about ``budget_s`` seconds (rope_theta: reconstruct-then-attend with
    that rotary base, else the latent decode's reference)."""
    run, n_max = _oracle_decode_case(cfg, rope_theta=rope_theta)
    P = cfg.page_tokens
    t0 = time.perf_counter()
    run(n_max)
    t_full = time.perf_counter() - t0
    per_step = budget_s / max(1, steps + warm)
    n_tok = int(n_max * per_step / max(t_full, 1e-9)) // P * P
    n_tok = max(P, min(n_max, n_tok))
    for _ in range(warm):
        run(n_tok)
    t0 = time.perf_counter()
    for _ in range(steps):
        run(n_tok)
    el = time.perf_counter() - t0
    value = steps * n_tok / el
    what = f"{steps} timed steps in {el:.1f} s"
    if rope_theta is not None:
        what += f", reconstruct-then-attend with rotary base {rope_theta:g}"
    return value, el / steps * 1e3, _blas_threads(), _sample_text(cfg, n_tok, what)


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
class ClockSampler:
    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        try:
            with open(self.path) as f:
                for line in f:
                    p = [x.strip() for x in line.split(",")]
                    if len(p) < 9:
                        continue
                    try:
                        sm.append(float(p[1]))
                        mx = float(p[2])
                    except ValueError:
                        continue
                    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
                    for nm, v in zip(names, p[5:9]):
                        if v.lower().startswith("active"):
                            reasons.add(nm)
        except OSError:
            pass
        finally:
            if self.path and os.path.exists(self.path):
                os.remove(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def _activation_source(cfg, dev, gen):
    """Seeded activations h = z sqrt(lambda) Q^T in the workload's basis (Gaussian,
    or multivariate Student-t when the workload says so), generated on the GPU."""
    import torch

    from workloads.synthetic import _basis
    basis = _basis(cfg.d_model, cfg.seed)
    lam = torch.arange(1, cfg.d_model + 1, device=dev, dtype=torch.float32) ** (-cfg.spectrum_exp)
    q1 = torch.from_numpy(basis[1]).to(dev, torch.float32)
    q2 = torch.from_numpy(basis[2]).to(dev, torch.float32) if basis[0] == "kron" else None

    def acts(n, seed):
        gen.manual_seed(seed)
        y = torch.randn((n, cfg.d_model), generator=gen, device=dev) * lam.sqrt()
        if q2 is None:
            h = y @ q1.T
        else:
            a, b = q1.shape[0], q2.shape[0]
            h = torch.einsum("ia,nab,jb->nij", q1, y.view(n, a, b), q2).reshape(n, a * b)
        if cfg.dist == "student_t":
            w = torch.distributions.Chi2(torch.tensor(cfg.nu, device=dev)).sample((n,))
            h = h * torch.sqrt(cfg.nu / w)[:, None]
        return h.to(torch.bfloat16)
    return acts


def _calibrated_codec(cfg, acts, gen, dev, layer):
    import torch

    import spectral_transform_coding_b200 as st
    from spectral_transform_coding_b200.codec import make_config
    c = make_config(cfg.d_model, cfg.n_q_heads, cfg.n_kv_heads, cfg.d_head, cfg.rank, cfg.group,
                    cfg.budget_bits, cfg.count_overhead, cfg.page_tokens)
    kvw = cfg.n_kv_heads * cfg.d_head
    gen.manual_seed(1000 * cfg.seed + layer)
    W_K = (torch.randn((cfg.d_model, kvw), generator=gen, device=dev) * cfg.w_std).to(torch.bfloat16)
    W_V = (torch.randn((cfg.d_model, kvw), generator=gen, device=dev) * cfg.w_std).to(torch.bfloat16)
    return st.Codec.calibrate(c, acts(cfg.calib_tokens, 7000 + layer), W_K, W_V)


def _launches_per_layer(B, rt):
    """Library kernels one layer of a decode step launches: the encode of B new
    tokens is one fused kernel for B <= 16 (projection, quantise, pack, append,
    length advance), else projection + append plan + quantise/pack; the latent
    decode is one kernel (query fold, split-K flash-decode, merge and W_up^V lift),
    reconstruct-then-attend is its split kernel and a combine kernel."""
    return (1 if B <= 16 else 3) + (2 if rt else 1)


def run_decode(args, name, world, local):
    """Decode steps through a stack of ``layers`` calibrated layers of workload
    ``name``; returns the JSON record of that workload."""
    import numpy as np
    import torch

    import spectral_transform_coding_b200 as st
    from workloads import get_config

    dev = torch.device("cuda", local)
    cfg = get_config(name)
    L = args.layers or MODEL_LAYERS[name]
    B = cfg.batch
    ctx = cfg.cache_len
    steps, warm = args.steps, args.warmup
    P = cfg.page_tokens
    ksteps_e2e = max(3, steps // 4)
    # every decode step appends one token per sequence: warm-up, timed, eager
    # end-to-end and graph end-to-end steps
    cap_tokens = ctx + warm + steps + 2 * ksteps_e2e + 8
    max_pages = (cap_tokens + P - 1) // P
    gen = torch.Generator(device=dev)
    acts = _activation_source(cfg, dev, gen)

    codecs, caches = [], []
    for l in range(L):
        codec = _calibrated_codec(cfg, acts, gen, dev, l)
        cache = st.LatentCache(codec, batch=B, max_pages_per_seq=max_pages, device=dev, zero=False)
        chunk = 8192
        for b in range(B):
            for t0 in range(0, ctx, chunk):
                n = min(chunk, ctx - t0)
                codec.encode_append(cache, acts(n, 10_000_000 + l * 1000 + b * 97 + t0 // chunk),
                                    torch.full((n,), b, dtype=torch.int32, device=dev))
        codec.device_status()
        codecs.append(codec)
        caches.append(cache)
    torch.cuda.synchronize()

    # per-step inputs and workspaces (device-resident)
    H_new = acts(L * B, 99).view(L, B, cfg.d_model).contiguous()
    gen.manual_seed(123)
    Q = (torch.randn((L, B, cfg.n_q_heads, cfg.d_head), generator=gen, device=dev) * 0.5).contiguous()
    OUT = torch.empty_like(Q)
    seq_ids = torch.arange(B, dtype=torch.int32, device=dev)
    ews = [torch.zeros(codecs[l].encode_workspace_bytes(B), dtype=torch.uint8, device=dev) for l in range(L)]
    rt = args.decode == "reconstruct"
    ws_bytes = (codecs[0].decode_reconstruct_workspace_bytes if rt else codecs[0].decode_workspace_bytes)
    dws = [torch.zeros(ws_bytes(B, cap_tokens), dtype=torch.uint8, device=dev) for l in range(L)]
    stream = torch.cuda.Stream(device=dev)

    def encode_layer(l):
        codecs[l].encode_append(caches[l], H_new[l], seq_ids, workspace=ews[l], stream=stream)

    def decode_layer(l):
        if rt:
            codecs[l].decode_attend_reconstruct(caches[l], Q[l], args.rope_theta, OUT[l], workspace=dws[l],
                                                stream=stream)
        else:
            codecs[l].decode_attend(caches[l], Q[l], OUT[l], workspace=dws[l], stream=stream)

    def step():
        for l in range(L):
            encode_layer(l)
            decode_layer(l)

    # host (pinned) buffers of the end-to-end arms: the step's new hidden states
    # and queries go up, its attention outputs come back
    H_host = H_new.cpu().pin_memory()
    Q_host = Q.cpu().pin_memory()
    OUT_host = torch.empty(OUT.shape, dtype=OUT.dtype).pin_memory()

    # Large per-step copies run on a second stream in slices of layers: every
    # slice of inputs goes up at once, a slice's layers start as soon as it has
    # landed, and its outputs come back while the next slice computes.  Small
    # ones (a few sequences) go in one piece on the compute stream, where the
    # events and extra copy calls would cost more than they hide.
    copy_stream = torch.cuda.Stream(device=dev)
    copy_bytes = (H_new.numel() * H_new.element_size() + Q.numel() * Q.element_size()
                  + OUT.numel() * OUT.element_size())
    n_slices = min(4, L) if copy_bytes >= (4 << 20) else 1
    cut = [round(i * L / n_slices) for i in range(n_slices + 1)]
    ev_start, ev_done = torch.cuda.Event(), torch.cuda.Event()
    ev_in = [torch.cuda.Event() for _ in range(n_slices)]
    ev_out = [torch.cuda.Event() for _ in range(n_slices)]

    def step_copies():
        if n_slices == 1:
            H_new.copy_(H_host, non_blocking=True)
            Q.copy_(Q_host, non_blocking=True)
            step()
            OUT_host.copy_(OUT, non_blocking=True)
            return
        ev_start.record(stream)
        copy_stream.wait_event(ev_start)  # the previous step is done with the device buffers
        with torch.cuda.stream(copy_stream):
            for k in range(n_slices):
                a, b = cut[k], cut[k + 1]
                H_new[a:b].copy_(H_host[a:b], non_blocking=True)
                Q[a:b].copy_(Q_host[a:b], non_blocking=True)
                ev_in[k].record(copy_stream)
        for k in range(n_slices):
            a, b = cut[k], cut[k + 1]
            stream.wait_event(ev_in[k])
            for l in range(a, b):
                encode_layer(l)
                decode_layer(l)
            ev_out[k].record(stream)
            copy_stream.wait_event(ev_out[k])
            with torch.cuda.stream(copy_stream):
                OUT_host[a:b].copy_(OUT[a:b], non_blocking=True)
        ev_done.record(copy_stream)
        stream.wait_event(ev_done)

    with torch.cuda.stream(stream):
        for _ in range(warm):
            step()
    torch.cuda.synchronize()
    len0 = int(caches[0].lengths.float().mean().item())

    # CUDA graphs: one decode step of all layers; decode attention of all layers;
    # the step with its host<->device copies
    g_step, g_dec, g_e2e = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_step, stream=stream):
        step()
    with torch.cuda.graph(g_dec, stream=stream):
        for l in range(L):
            decode_layer(l)
    with torch.cuda.graph(g_e2e, stream=stream):
        step_copies()
    torch.cuda.synchronize()
    for codec in codecs:
        codec.device_status()

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    def timed(body, n):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            a.record(stream)
            for _ in range(n):
                body()
            b.record(stream)
        torch.cuda.synchronize()
        barrier()
        return a.elapsed_time(b)

    def eager_e2e():
        # one step as a user runs it: eager calls through the C ABI for every
        # layer, inputs copied up from host memory, outputs read back on the host
        step_copies()
        stream.synchronize()

    # ---- device-resident timed region: K decode steps ----
    with ClockSampler(local) as clocks:
        total_ms = timed(g_step.replay, steps)
    clk = clocks.summary()
    len_after = int(caches[0].lengths.float().mean().item())
    # ---- decode-attention launches alone (same kernels, same resident caches) ----
    dec_ms = timed(g_dec.replay, steps) / (steps * L)
    # ---- end to end: eager per-step calls with host buffers; graph replay of the same ----
    e2e_ms = timed(eager_e2e, ksteps_e2e) / ksteps_e2e
    e2e_graph_ms = timed(g_e2e.replay, ksteps_e2e) / ksteps_e2e
    for codec in codecs:
        codec.device_status(stream)
    ms_per_step = total_ms / steps
    if world > 1:
        ms_per_step, e2e_ms, e2e_graph_ms, dec_ms = max_over_ranks([ms_per_step, e2e_ms, e2e_graph_ms, dec_ms], dev)
    mean_ctx = (len0 + len_after) / 2.0
    tok_per_step = L * B * mean_ctx * cfg.n_kv_heads
    value = replicas_throughput(tok_per_step, ms_per_step, world)
    e2e_value = replicas_throughput(tok_per_step, e2e_ms, world)
    e2e_graph_value = replicas_throughput(tok_per_step, e2e_graph_ms, world)

    # roofline of the decode kernel: the packed bytes one launch must read (every
    # token of every sequence of the layer, all KV heads) over its average launch
    # time, launches timed back to back over resident caches of all layers
    bytes_per_tok_all_heads = codecs[0].page_bytes / P
    dec_bytes = B * len_after * bytes_per_tok_all_heads
    peaks = _peaks()
    achieved = dec_bytes / (dec_ms / 1e3) / 1e9
    h2d = H_new.numel() * H_new.element_size() + Q.numel() * Q.element_size()
    d2h = OUT.numel() * OUT.element_size()
    check = _self_check(codecs[0], caches[0], Q[0], OUT[0], stream) if args.check else None

    result = {
        "metric": "latent-KV decode attention: cache tokens/s/head",
        "value": value,
        "unit": "tokens/s/head",
        "n_gpus": world,
        "steps": steps,
        "warmup": warm,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "u8 codes, fp16 scale/zero, fp32 accumulate",
        "data": "synthetic (seeded power-law activations, random bf16 weights; calibrated per layer)",
        "config": {
            "workload": _workload_name(cfg, L),
            "layers": L, "batch": B, "context_start": len0, "n_kv_heads": cfg.n_kv_heads,
            "bytes_per_token_per_layer": bytes_per_tok_all_heads,
            "l2": "inputs larger than L2 (caches + factors of all layers)",
            "parallelism": f"replicas x{world}",
        },
        "roofline": {
            "kernel": "attend_kernel (query fold, split-K latent flash-decode over the packed pages, "
                      "last-CTA merge and W_up^V lift in one launch)",
            "bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / peaks["hbm_gbs"],
            "traffic": (TRAFFIC_PER_ALGO_BYTE[name] * dec_bytes if name in TRAFFIC_PER_ALGO_BYTE else None),
            "peak_src": peaks["src"], "avg_launch_us": dec_ms * 1e3,
            "algorithmic_bytes_per_launch": dec_bytes,
            "timing": "decode launches of all layers replayed back to back (CUDA graph, PDL chained), "
                      "CUDA events on the launching stream",
        },
        "e2e": {"value": e2e_value, "unit": "tokens/s/head", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "how": "eager per-step calls through the C ABI (encode_append + decode_attend per layer), "
                       "inputs copied from pinned host memory, outputs copied back and the host synchronised "
                       "on them every step" + ("; the copies run on a second stream in slices of layers, "
                                                 "overlapping the other slices' kernels" if n_slices > 1 else "")},
        "e2e_graph": {"value": e2e_graph_value, "unit": "tokens/s/head", "ms_per_step": e2e_graph_ms,
                      "how": "the same step with its copies captured once in a CUDA graph and replayed"},
        "gpu_launches": _launches_per_layer(B, rt) * L * steps,
        "clocks": clk,
    }
    if check is not None:
        result["check"] = check
    if rt:
        # Two pipes.  CUDA cores: per (token, KV head) the rotation (6 FLOP per pair
        # of dims = 3 d_h), the scores 2 gq d_h and the probability-weighted V
        # latents 2 gq n_kept_V, against the fp32 peak.  Tensor cores: the key lift
        # 2 n_kept_K d_h, issued as two fp16 MMAs (hi and lo parts of W_up^K), i.e.
        # 4 n_kept_K d_h MMA FLOPs, against the bf16/fp16 dense peak.  The kernel's
        # time bound is the larger of the two times; it is far above both (issue-
        # and latency-bound per-tile phases).
        widths = codecs[0].state()["widths"]
        gq = cfg.n_q_heads // cfg.n_kv_heads
        alu_tok = sum(3 * cfg.d_head + 2 * gq * cfg.d_head + 2 * gq * cfg.group * int((w[1] > 0).sum())
                      for w in widths)
        mma_tok = sum(4 * cfg.group * int((w[0] > 0).sum()) * cfg.d_head for w in widths)
        alu_flops = B * len_after * alu_tok
        mma_flops = B * len_after * mma_tok
        alu_peak = 148 * 128 * 2 * 1965e6 / 1e12
        t_s = dec_ms / 1e3
        alu_tflops = alu_flops / t_s / 1e12
        mma_tflops = mma_flops / t_s / 1e12
        bound_s = max(alu_flops / (alu_peak * 1e12), mma_flops / (peaks["bf16_tflops"] * 1e12))
        result["config"]["decode"] = f"reconstruct-then-attend, rotary base {args.rope_theta:g}"
        result["dtype"] = "u8 codes, fp16 scale/zero, fp32 lift and accumulate"
        result["roofline"] = {
            "kernel": "rt_split_kernel (keys rebuilt per 32-token tile on the tensor cores, rotated and scored "
                      "with fp32 FMAs; V summed in the latent space), timed with its combine launch",
            "bound": "alu", "achieved": alu_tflops, "peak": alu_peak, "unit": "TFLOP/s",
            "frac": alu_tflops / alu_peak,
            "traffic": (TRAFFIC_PER_PACKED_BYTE_RT[name] * dec_bytes if name in TRAFFIC_PER_PACKED_BYTE_RT
                        else None),
            "peak_src": "derived: 148 SMs x 128 fp32 lanes x 2 FLOP x 1965 MHz (clocks.max.sm); CUDA-core FLOPs only",
            "avg_launch_us": dec_ms * 1e3, "cuda_core_flops_per_launch": alu_flops,
            "tensor": {"mma_flops_per_launch": mma_flops, "tflops": mma_tflops, "peak": peaks["bf16_tflops"],
                       "frac": mma_tflops / peaks["bf16_tflops"]},
            "time_bound_us": bound_s * 1e6, "time_bound_frac": bound_s / t_s,
            "packed_bytes_per_launch": dec_bytes,
            "hbm_gbs": achieved, "hbm_frac": achieved / peaks["hbm_gbs"],
        }
    del g_step, g_dec, g_e2e, codecs, caches
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return result


def _self_check(codec, cache, q, out, stream):
    """Opt-in self-consistency check after timing: the latent decode of layer 0
    against reconstruct-then-attend without rotation over the same pages (a second
    kernel that rebuilds keys and values from the codes and attends over them; the
    two agree to rounding).  The element-wise checks against the CPU oracle at
    these shapes live in the GPU test suite."""
    import torch
    torch.cuda.synchronize()
    a = codec.decode_attend(cache, q)
    b = codec.decode_attend_reconstruct(cache, q, rope_theta=0.0)
    codec.device_status()
    a64, b64 = a.double(), b.double()
    err = ((a64 - b64).abs().amax(dim=-1) / b64.abs().amax(dim=-1).clamp_min(1e-30)).max().item()
    return {"what": "layer 0: latent decode vs reconstruct-then-attend (no rotation), all sequences and q heads",
            "max_rel_err": err, "bar": 2e-3, "ok": bool(err <= 2e-3)}


def run_prefill(args, local):
    """Prefill encode of one 65,536-token bf16 chunk for all KV heads of the
    Llama-shaped layer at 4x and 8x, then one decode step over it.  Per budget:
    encode tokens/s and TFLOP/s (projection GEMM with the quantiser in its
    epilogue), for comparison the projection alone and the separate quantise/pack
    kernel on its fp32 latents, and the decode after it."""
    import torch

    import spectral_transform_coding_b200 as st
    from workloads import get_config

    dev = torch.device("cuda", local)
    peaks = _peaks()
    out = []
    for name in ("prefill", "prefill8"):
        cfg = get_config(name)
        T, P = args.prefill_tokens or cfg.prefill_tokens, cfg.page_tokens
        gen = torch.Generator(device=dev)
        acts = _activation_source(cfg, dev, gen)
        codec = _calibrated_codec(cfg, acts, gen, dev, 0)
        H = acts(T, 12345)
        cache = st.LatentCache(codec, batch=1, max_pages_per_seq=(T + P - 1) // P + 1, device=dev, zero=False)
        seq = torch.zeros(T, dtype=torch.int32, device=dev)
        ws = torch.zeros(codec.encode_workspace_bytes(T), dtype=torch.uint8, device=dev)
        lat = torch.empty((T, codec.n_eff), dtype=torch.float32, device=dev)
        stream = torch.cuda.Stream(device=dev)
        gen.manual_seed(77)
        q = (torch.randn((1, cfg.n_q_heads, cfg.d_head), generator=gen, device=dev) * 0.5).contiguous()
        o = torch.empty_like(q)
        dws = torch.zeros(codec.decode_workspace_bytes(1, cache.capacity), dtype=torch.uint8, device=dev)

        def timed(fn, reps):
            # each repetition encodes the chunk into an emptied cache; the chunk and
            # its latents (0.5 + 0.5 GB at 4x) exceed L2
            tot = 0.0
            for r in range(reps + 3):
                cache.lengths.zero_()
                torch.cuda.synchronize()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                with torch.cuda.stream(stream):
                    e0.record(stream)
                    fn()
                    e1.record(stream)
                torch.cuda.synchronize()
                if r >= 3:
                    tot += e0.elapsed_time(e1)
            return tot / reps

        reps = max(3, min(args.steps, 10))
        with ClockSampler(local) as clocks:
            t_enc = timed(lambda: codec.encode_append(cache, H, seq, workspace=ws, stream=stream), reps)
            t_proj = timed(lambda: codec.project(H, out=lat, stream=stream), reps)
            t_quant = timed(lambda: codec.quantize_append(cache, lat, seq, workspace=ws, stream=stream), reps)
        clk = clocks.summary()
        cache.lengths.zero_()
        codec.encode_append(cache, H, seq, workspace=ws, stream=stream)  # leave the cache full for decode
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            for _ in range(3):
                codec.decode_attend(cache, q, o, workspace=dws, stream=stream)
            e0.record(stream)
            for _ in range(10):
                codec.decode_attend(cache, q, o, workspace=dws, stream=stream)
            e1.record(stream)
        torch.cuda.synchronize()
        t_dec = e0.elapsed_time(e1) / 10
        codec.device_status(stream)
        flops = 2.0 * cfg.d_model * codec.n_eff * T
        packed = T * codec.page_bytes / P
        qbytes = T * 4.0 * codec.n_eff + packed
        bf16 = peaks["bf16_tflops"]
        out.append({
            "metric": "prefill encode-append tokens/s", "value": T / (t_enc / 1e3), "unit": "tokens/s",
            "workload": f"{name}: {T} tokens x (d_model {cfg.d_model}, {cfg.n_kv_heads} kv heads, "
                        f"{cfg.budget_bits} bits/side), one chunk, then one decode step",
            "n_eff": codec.n_eff, "packed_bytes": packed,
            "encode": {"ms": t_enc, "tflops": flops / (t_enc / 1e3) / 1e12, "peak": bf16,
                       "frac": flops / (t_enc / 1e3) / 1e12 / bf16, "latent_bytes_written": 0,
                       "kernels": "append_plan_kernel, then encode_gemm_kernel (tcgen05 projection with "
                                  "quantise/pack/append in its epilogue)"},
            "projection_only": {"ms": t_proj, "tflops": flops / (t_proj / 1e3) / 1e12, "peak": bf16,
                                "frac": flops / (t_proj / 1e3) / 1e12 / bf16,
                                "kernel": "gemm_tcgen05_kernel (bf16 in, fp32 latents out)"},
            "unfused_quantize_pack": {"ms": t_quant, "gbs": qbytes / (t_quant / 1e3) / 1e9, "peak": peaks["hbm_gbs"],
                                      "frac": qbytes / (t_quant / 1e3) / 1e9 / peaks["hbm_gbs"], "bytes": qbytes,
                                      "kernels": "append_plan_kernel + quantize_append_kernel on fp32 latents"},
            "decode_after_us": t_dec * 1e3, "peak_src": peaks["src"], "clocks": clk,
        })
        del codec, cache, H, lat, ws, dws
        torch.cuda.empty_cache()
    return out


def _reference_line(args, name):
    """The CPU oracle as the reference arm on ``name``'s configuration."""
    from workloads import get_config
    cfg = get_config(name)
    rt = args.decode == "reconstruct"
    value, ms, cores, sample = cpu_oracle_steps(cfg, args.steps, args.warmup,
                                                rope_theta=args.rope_theta if rt else None)
    L = args.layers or MODEL_LAYERS[name]
    return {
        "impl": "reference", "metric": "latent-KV decode attention: cache tokens/s/head", "value": value,
        "unit": "tokens/s/head", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": dict({"workload": _workload_name(cfg, L)},
                       **({"decode": f"reconstruct-then-attend, rotary base {args.rope_theta:g}"} if rt else {})),
        "cpu_baseline": {"value": value, "unit": "tokens/s/head", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s/head", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="stress", choices=sorted(MODEL_LAYERS),
                    help="the workload of the line's top-level figures")
    ap.add_argument("--extra", default="qwen,llama,prefill",
                    help="comma-separated workloads measured after it and nested in the same line "
                         "(decode workloads and/or 'prefill'; empty for none)")
    ap.add_argument("--layers", type=int, default=0, help="layers per decode workload (default: the model's)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--check", action="store_true",
                    help="after timing, check layer 0's decode against reconstruct-then-attend")
    ap.add_argument("--decode", default="latent", choices=["latent", "reconstruct"],
                    help="decode attention: in the latent space (default) or over keys rebuilt per tile")
    ap.add_argument("--rope-theta", type=float, default=500000.0,
                    help="reconstruct decode: rotary base (0 = no rotation)")
    ap.add_argument("--prefill-tokens", type=int, default=0,
                    help="prefill: tokens in the chunk (default: the workload's 65,536)")
    args = ap.parse_args()
    if args.impl == "ours" and args.warmup < 3:
        ap.error("--warmup must be at least 3")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    extras = [e for e in args.extra.split(",") if e]
    for e in extras:
        if e != "prefill" and e not in MODEL_LAYERS:
            ap.error(f"unknown workload {e!r}")

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(_reference_line(args, args.workload)), flush=True)
        return 0

    from workloads import get_config
    import torch
    torch.cuda.set_device(local)
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_oracle_sample(get_config(args.workload),
                                rope_theta=args.rope_theta if args.decode == "reconstruct" else None)
    res = run_decode(args, args.workload, world, local)
    nested = {}
    for e in extras:
        if e == "prefill":
            nested["prefill"] = run_prefill(args, local)
        elif e != args.workload:
            r = run_decode(args, e, world, local)
            nested[e] = {k: r[k] for k in ("value", "unit", "ms_per_step", "config", "roofline", "e2e",
                                           "e2e_graph", "gpu_launches", "clocks", "check") if k in r}
    if rank == 0:
        if cpu is not None:
            res["cpu_baseline"] = {"value": cpu[0], "unit": "tokens/s/head", "cores": cpu[1], "kind": "oracle",
                                   "sample": cpu[2]}
        if nested:
            res["workloads"] = nested
        print(json.dumps(res), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
