"""Benchmark of the Zebra3D hybrid global-attention layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload views1024] [--impl reference]

One step = one pass of the whole hot path on one synthetic 1,024-view input
(16 heads x 1,406,976 tokens, d = 64, bf16): the tile-sparse stage (landmark
means, fp64 tile selection keeping 6% of key tiles, tile-sparse attention with
landmarks) and the linear stage (elu+1 state, dense attention on 4,096
calibration rows, closed-form affine fit, fitted linear attention on all
rows).  The metric is hybrid-layer throughput with half the layers linear
(0.5L): tokens / (0.5 t_linear + 0.5 t_sparse) = 2 N / t_step, in Mtokens/s.

Prints ONE JSON line on rank 0.  Under torchrun every rank runs its own
independent input (weak scaling, no collective on the data path).
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
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import synth  # noqa: E402
from linear_hybrid_attention_b200 import replicas  # noqa: E402

METRIC = "hybrid global-attn layer Mtokens/s at 1,024 views; % bf16 TC peak / % HBM BW"
UNIT = "Mtokens/s"


# ------------------------------------------------------------------ peaks ----
def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ---------------------------------------------------------------- traffic ----
def recorded_traffic(workload: str):
    """DRAM bytes per launch of the sparse kernel at this workload, from the small
    record profiles/sparse_attn_<workload>_traffic.json written beside the ncu
    summary it comes from, or None when there is none or when the kernel source
    changed since the capture (the record holds attn.cu's sha256)."""
    import hashlib
    path = os.path.join(ROOT, "profiles", f"sparse_attn_{workload}_traffic.json")
    src = os.path.join(ROOT, "linear_hybrid_attention_b200", "csrc", "attn.cu")
    if not os.path.exists(path) or not os.path.exists(src):
        return None, "no ncu DRAM capture recorded for this workload"
    with open(path) as f:
        rec = json.load(f)
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()
    if rec.get("attn_cu_sha256") != sha:
        return None, "kernel changed since the recorded ncu DRAM capture"
    return float(rec["dram_bytes_per_launch"]), rec.get("summary", os.path.relpath(path, ROOT))


# ----------------------------------------------------------------- clocks ----
class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons during the timed region."""

    FIELDS = ("index,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.path = None
        try:
            props = torch.cuda.get_device_properties(device_index)
            u = str(getattr(props, "uuid", ""))
            self.uuid = u if u.startswith("GPU-") else ("GPU-" + u if u else "")
        except Exception:
            self.uuid = ""

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200"]
            if self.uuid:
                cmd += ["-i", self.uuid]
            self.proc = subprocess.Popen(cmd, stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        try:
            with open(self.path) as f:
                for line in f:
                    parts = [p.strip() for p in line.split(",")]
                    if len(parts) >= 10:
                        rows.append(parts)
            os.remove(self.path)
        except Exception:
            return None
        if not rows:
            return None
        sm = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        smax = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[6 + i].lower().startswith("active")})
        loaded = [s for s in sm if smax and s > 0.5 * max(smax)] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------ L2 / HBM ----
L2_FLUSH_BYTES = 256 << 20   # twice the B200's 126 MB L2
SPEC_HBM_GBS = 7700.0        # nominal HBM3e bandwidth of an HGX B200


class L2Flush:
    """Writes a buffer twice the size of L2, evicting whatever an earlier call left there."""

    def __init__(self, device):
        self.buf = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=device)

    def __call__(self):
        self.buf.fill_(1)


def read_stream_gbs(device, gib: int = 4, reps: int = 5) -> float:
    """Read-dominated HBM rate: a sum over a buffer far larger than L2 (the
    driver's peak is a copy, half writes), with L2 flushed between repetitions."""
    x = torch.ones(gib << 28, dtype=torch.float32, device=device)
    flush = L2Flush(device)
    x.sum()
    times = []
    for _ in range(reps):
        flush()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        x.sum()
        b.record()
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b) / 1e3)
    nbytes = x.numel() * 4
    del x, flush
    return nbytes / min(times) / 1e9


def hbm_isolated(fns: dict, device, local_rank: int, seconds: float = 0.5) -> dict:
    """Each HBM kernel alone: launched back to back for about `seconds` (L2 flushed
    before every launch), CUDA events around each launch, nvidia-smi clocks sampled
    over the whole loop.  Returns the median ms of each and the clock record."""
    flush = L2Flush(device)
    for fn in fns.values():
        fn()
    torch.cuda.synchronize()
    clocks = ClockSampler(local_rank)
    clocks.start()
    out = {}
    for name, fn in fns.items():
        evs = []
        t0 = time.time()
        while time.time() - t0 < seconds:
            for _ in range(20):
                flush()
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record()
                fn()
                b.record()
                evs.append((a, b))
            torch.cuda.synchronize()
        out[name] = statistics.median(a.elapsed_time(b) for a, b in evs)
    clk = clocks.stop()
    del flush
    return {"ms": out, "clocks": clk}


def cpu_model() -> str:
    """The host CPU's model name (from /proc/cpuinfo), for the CPU baseline's record."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.lower().startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


# --------------------------------------------------------------- CPU oracle ----
def oracle_sample(w, Q, K, V, calib_tiles, sample_tiles=4, calib_rows=16, head=0):
    """Time the fp64 oracle on a bounded sample of one head and extrapolate.

    Fixed per-head work (landmark means, linear state, calibration dense rows +
    unfitted linear rows + fit) and per-query-tile work (selection row, sparse
    attention, fitted linear output) are timed on `sample_tiles` query tiles and
    `calib_rows` calibration rows of one head, then scaled to the full job.
    Returns (extrapolated seconds per step, description, cores)."""
    import oracle
    cores = len(os.sched_getaffinity(0))
    d = w.head_dim
    s = 1.0 / math.sqrt(d)
    t0 = time.perf_counter()
    q = synth.to_f64(Q[head:head + 1])
    k = synth.to_f64(K[head:head + 1])
    v = synth.to_f64(V[head:head + 1])
    t_load = time.perf_counter() - t0
    # --- fixed per-head work
    t0 = time.perf_counter()
    Qb = oracle.landmark_means(q, w.tile)
    Kb = oracle.landmark_means(k, w.tile)
    S, z = oracle.linear_state(k, v)
    t_fixed = time.perf_counter() - t0
    rows = oracle.calibration_rows(w.n_tokens, w.tile, calib_tiles)
    sub = rows[:calib_rows]
    t0 = time.perf_counter()
    Y = np.concatenate([oracle.dense_attention(q[:, sub[c:c + 16]], k, v, s)
                        for c in range(0, len(sub), 16)], axis=1)
    X = oracle.linear_attention(q[:, sub], k, v)
    t_cal = (time.perf_counter() - t0) * (len(rows) / len(sub))
    # the fit itself is timed at the full calibration size (the values of the
    # tiled rows do not matter for its cost; a small jitter keeps it full-rank)
    reps = -(-len(rows) // len(sub))
    jit = 1e-3 * np.random.default_rng(0).standard_normal((1, len(rows), d))
    Xf = np.tile(X, (1, reps, 1))[:, : len(rows)] + jit
    Yf = np.tile(Y, (1, reps, 1))[:, : len(rows)]
    t0 = time.perf_counter()
    A, b = oracle.affine_fit(Xf, Yf)
    t_fit = time.perf_counter() - t0
    # --- per-query-tile work
    tiles = list(np.linspace(0, w.n_tiles - 1, sample_tiles).astype(int))
    t0 = time.perf_counter()
    sc = oracle.tile_scores(Qb[:, tiles], Kb)
    idx_s = oracle.select_tiles(sc, w.k)
    idx = np.zeros((1, w.n_tiles, w.k), dtype=np.int64)
    idx[0, tiles] = idx_s[0]
    oracle.sparse_attention(q, k, v, w.tile, idx, s, query_tiles=tiles)
    qrows = oracle.calibration_rows(w.n_tokens, w.tile, tiles)
    oracle.linear_apply(q[:, qrows], S, z, A, b)
    t_tiles = time.perf_counter() - t0
    per_head = t_fixed + t_cal + t_fit + t_tiles * (w.n_tiles / sample_tiles)
    total = per_head * w.heads
    desc = (f"fp64 oracle on head {head}: landmarks + linear state of the head, {len(sub)} of {len(rows)} "
            f"calibration rows, {sample_tiles} of {w.n_tiles} query tiles (selection, sparse attention, "
            f"fitted linear); extrapolated to {w.heads} heads x {w.n_tiles} tiles "
            f"(sample time {t_fixed + t_cal / (len(rows) / len(sub)) + t_fit + t_tiles:.1f} s, "
            f"load {t_load:.1f} s)")
    return total, desc, cores


# ------------------------------------------------------------------- main ----
def landmark_flops(heads: int, n_tokens: int, n_tiles_: int, k: int, d: int) -> float:
    """4 * d per (query row, landmark): every row attends to the T - k landmarks of its
    omitted tiles (logit q . Kbar_j and the product with Vbar_j)."""
    return float(4.0 * d * heads * n_tokens * (n_tiles_ - k))


def selected_flops(idx_cpu: np.ndarray, n_tokens: int, tile: int, d: int) -> float:
    """4 * d * sum over (h, i, j in sel) n_i * n_j: the algorithmic FLOPs of QK^T and PV."""
    T = idx_cpu.shape[1]
    n = np.full(T, tile, dtype=np.float64)
    n[-1] = n_tokens - (T - 1) * tile
    per_row = n[idx_cpu].sum(axis=-1)  # [H, T]
    return float(4.0 * d * (per_row * n[None, :]).sum())


def run_reference(args, w):
    rank, _, world = replicas.env_rank()
    if rank != 0:
        return 0
    Q, K, V = synth.make_qkv(w, device="cpu" if not torch.cuda.is_available() else "cuda")
    calib = synth.calibration_tiles(w.n_tiles, w.calib_tiles)
    times = []
    desc = cores = None
    for _ in range(args.warmup + args.steps):
        t, desc, cores = oracle_sample(w, Q, K, V, calib, sample_tiles=2, calib_rows=8)
        times.append(t)
    t = statistics.median(times[args.warmup:]) if args.steps else times[-1]
    value = 2 * w.n_tokens / t / 1e6
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_dict(w),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "cpu_model": cpu_model(), "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def linear_centered_report(zb, w, layer, Q, K, V, stream, hbm, tensor_bytes, t_apply):
    H, N, d = w.heads, w.n_tokens, w.head_dim
    dev = Q.device
    mu = torch.empty(H, d, dtype=torch.float32, device=dev)
    ws_km = torch.empty(max(zb.key_mean_workspace_bytes(H, N, d), 16), dtype=torch.uint8, device=dev)
    S_c = torch.empty_like(layer.S)
    z_c = torch.empty_like(layer.z)

    def centred_state(ev=None):
        if ev is not None:
            ev[0].record(stream)
        zb.zb_key_mean(K, out=mu, ws=ws_km)
        if ev is not None:
            ev[1].record(stream)
        zb.zb_linear_state_centered(K, V, mu, S_c, z_c, layer.ws_lin)
        if ev is not None:
            ev[2].record(stream)

    centred_state()
    torch.cuda.synchronize()
    reps = 5
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(reps)]
    flush = L2Flush(Q.device)
    for ev in evs:
        flush()
        centred_state(ev)
    torch.cuda.synchronize()
    zb.zb_last_device_status()
    t_km = statistics.mean(ev[0].elapsed_time(ev[1]) for ev in evs) / 1e3
    t_sc = statistics.mean(ev[1].elapsed_time(ev[2]) for ev in evs) / 1e3

    # fit on the calibration rows (the step's dense rows Yc), then residuals of the
    # fitted outputs, all computed by the library's kernels
    Xc_c = torch.empty_like(layer.Xc)
    zb.zb_linear_apply(layer.Qc, S_c, z_c, None, None, out=Xc_c, out_fp32=True)
    A_c, b_c = zb.zb_affine_fit(Xc_c, layer.Yc, ws=layer.ws_fit)
    T = w.n_tiles
    m = len(layer.calib)
    held = sorted({int((i + 0.5) * T / m) for i in range(m)} - set(layer.calib.tolist()) - {T - 1})
    held_t = torch.as_tensor(held, dtype=torch.int32, device=dev)
    Qh = zb.zb_gather_tiles(Q, w.tile, held_t)
    Yh = zb.zb_dense_attn(Qh, K, V, layer.scale, out_fp32=True)

    def resid(Qr, Y, S, z, A, b):
        fit = zb.zb_linear_apply(Qr, S, z, A, b, out_fp32=True)
        num = (fit - Y).double().flatten(1).norm(dim=1)
        return float((num / Y.double().flatten(1).norm(dim=1)).max())

    res = {"calibration_rows": {"uncentered": resid(layer.Qc, layer.Yc, layer.S, layer.z, layer.A, layer.b),
                                "centered": resid(layer.Qc, layer.Yc, S_c, z_c, A_c, b_c)},
           "held_out_rows": {"uncentered": resid(Qh, Yh, layer.S, layer.z, layer.A, layer.b),
                             "centered": resid(Qh, Yh, S_c, z_c, A_c, b_c)}}
    torch.cuda.synchronize()
    zb.zb_last_device_status()
    return {"zb_key_mean": {"bound": "hbm", "ms": t_km * 1e3, "achieved": tensor_bytes / t_km / 1e9, "peak": hbm,
                            "unit": "GB/s", "frac": tensor_bytes / t_km / 1e9 / hbm},
            "zb_linear_state_centered": {"bound": "hbm", "ms": t_sc * 1e3, "achieved": 2 * tensor_bytes / t_sc / 1e9,
                                         "peak": hbm, "unit": "GB/s", "frac": 2 * tensor_bytes / t_sc / 1e9 / hbm},
            "stage_ms_without_fit": (t_km + t_sc + t_apply) * 1e3,
            "fit_residual": res,
            "held_out_rows": len(held) * w.tile,
            "note": "max over heads of |fitted linear output - dense output|_F / |dense output|_F; "
                    "synthetic random inputs, not a trained model's activations"}


def block_mass_report(zb, w, layer, Q, K, V, stream):
    """Dense-softmax mass kept by selections, on head 0 (the heads are alike):
    the heaviest 20% of 64 x 64 blocks, the heaviest 20% and the heaviest k of
    the tiles, and the method's own k selected tiles (mean-pooled scores)."""
    q1, k1, v1 = Q[:1], K[:1], V[:1]
    _, lse = zb.zb_dense_attn(q1, k1, v1, layer.scale, want_lse=True)
    M64 = zb.zb_block_mass(q1, k1, lse, 64, layer.scale)
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    bb = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    zb.zb_block_mass(q1, k1, lse, 64, layer.scale, out=M64)
    bb.record(stream)
    torch.cuda.synchronize()
    t = a.elapsed_time(bb) / 1e3
    T64 = M64.shape[-1]
    top64 = zb.zb_block_mass_top_fraction(M64, math.ceil(0.2 * T64))
    Mt = zb.zb_block_mass(q1, k1, lse, w.tile, layer.scale)
    T = Mt.shape[-1]
    top_t20 = zb.zb_block_mass_top_fraction(Mt, math.ceil(0.2 * T))
    top_tk = zb.zb_block_mass_top_fraction(Mt, w.k)
    sel = zb.zb_block_mass_selected_fraction(Mt, layer.idx[:1].contiguous())
    torch.cuda.synchronize()
    zb.zb_last_device_status()
    n = w.n_tokens
    exps = float(n) * n
    mufu_bound = 16.0 * torch.cuda.get_device_properties(Q.device).multi_processor_count * 1.965e9
    out = {"head": 0, "block_mass_64_ms": t * 1e3, "qk_tflops": 2.0 * n * n * w.head_dim / t / 1e12,
           "exp_per_s": exps / t, "frac_of_mufu_bound": exps / t / mufu_bound,
           "mufu_bound_note": "16 exponentials per clock per SM at the 1,965 MHz maximum clock",
           "retained_mass": {"top20pct_64x64_blocks": float(top64.mean()),
                             f"top20pct_{w.tile}_tiles": float(top_t20.mean()),
                             f"top{w.k}_{w.tile}_tiles": float(top_tk.mean()),
                             f"method_selected_{w.k}_tiles": float(sel.mean())},
           "note": "mean over query blocks of head 0; synthetic inputs with planted tiles"}
    del M64, Mt
    return out


def stack_report(zb, rank, dev, stream, passes=2):
    """The 512-view stack: 24 freshly seeded layers (12 linear at VGGT's 0.5L
    positions, 12 tile-sparse keeping 20% of the tiles), all inputs resident
    (24 x 3 x 1.44 GB), run by HybridStack.  Reports one serial pass with
    per-layer events (the sum of the parts) and `passes` timed passes with the
    next layer's input side issued ahead on a second stream."""
    from linear_hybrid_attention_b200.stack import HybridStack
    w = synth.WORKLOADS["stack512"]
    L = w.layers
    inputs = [synth.make_qkv(w, layer=l, device=dev,
                             seed=replicas.rank_seed(synth.default_seed(w, layer=l), rank)) for l in range(L)]
    calib = synth.calibration_tiles(w.n_tiles, w.calib_tiles)
    stack = HybridStack(w.heads, w.n_tokens, w.tile, w.k, calib, L, w.linear_layers, device=dev)
    stack.run(inputs)                                     # warm-up
    torch.cuda.synchronize()
    zb.zb_last_device_status()
    lev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(L)]
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    stack.run(inputs, lookahead=False, layer_events=lev)
    b.record(stream)
    torch.cuda.synchronize()
    serial_ms = a.elapsed_time(b)
    per_layer = [e0.elapsed_time(e1) for e0, e1 in lev]
    a.record(stream)
    for _ in range(passes):
        stack.run(inputs)
    b.record(stream)
    torch.cuda.synchronize()
    zb.zb_last_device_status()
    ahead_ms = a.elapsed_time(b) / passes
    lin = [per_layer[l] for l in range(L) if l in stack.linear]
    sp = [per_layer[l] for l in range(L) if l not in stack.linear]
    out = {"workload": f"stack512: 24 layers (linear at {list(w.linear_layers)}, the others tile-sparse keeping "
                       f"{w.k}/{w.n_tiles} tiles + landmarks), each freshly seeded; 16 heads x {w.n_tokens} tokens",
           "mtokens_s": w.n_tokens / (ahead_ms / 1e3) / 1e6,
           "ms_per_pass": ahead_ms, "passes": passes,
           "serial_pass_ms": serial_ms, "sum_of_layers_ms": sum(per_layer),
           "lookahead_saved_ms": serial_ms - ahead_ms,
           "per_layer_ms": [round(x, 3) for x in per_layer],
           "sparse_layer_ms_mean": statistics.mean(sp), "linear_layer_ms_mean": statistics.mean(lin),
           "gpu_launches_per_pass": stack.launches(),
           "note": "Mtokens/s = tokens through all 24 layers / time of one pass; linear layers include "
                   "their calibration (dense rows + fit); inputs resident in HBM"}
    del stack, inputs
    torch.cuda.empty_cache()
    return out


def spatial_report(zb, dev, stream):
    """Spatial tiles on the 32-view recipe with 2-D positional locality (16 heads,
    k = 69 of 344 tiles): time of the tile-sparse stage with the tokens reordered
    into 8 x 16 patch windows (gathers in and out included) against the plain
    stage, and the dense-softmax mass each tiling keeps on head 0: the heaviest
    k tiles, and the k tiles the method selects."""
    w = synth.WORKLOADS["spatial32"]
    views = w.n_tokens // synth.TOKENS_PER_VIEW
    Q, K, V = synth.make_qkv(w, device=dev)
    geom = (views, synth.GRID, synth.SPECIALS, 8, 16)
    plain = zb.HybridLayer(w.heads, w.n_tokens, w.tile, w.k, [0], device=dev)
    spat = zb.HybridLayer(w.heads, w.n_tokens, w.tile, w.k, [0], device=dev, spatial=geom)
    out = {"workload": f"spatial32: {views} views x {synth.TOKENS_PER_VIEW} tokens, 16 heads, keep {w.k}/{w.n_tiles} "
                       f"tiles; queries and keys carry a 2-D positional component (scale {w.pos_scale}, length "
                       f"{w.pos_length} patches)", "windows": "8 x 16 patches"}
    for name, layer in (("row_major_tiles", plain), ("window_tiles", spat)):
        layer.sparse(Q, K, V)
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(3):
            layer.sparse(Q, K, V)
        b.record(stream)
        torch.cuda.synchronize()
        zb.zb_last_device_status()
        q1 = (layer.Qp if layer.spatial else Q)[:1].contiguous()
        k1 = (layer.Kp if layer.spatial else K)[:1].contiguous()
        v1 = (layer.Vp if layer.spatial else V)[:1].contiguous()
        _, lse = zb.zb_dense_attn(q1, k1, v1, layer.scale, want_lse=True)
        M = zb.zb_block_mass(q1, k1, lse, w.tile, layer.scale)
        top = zb.zb_block_mass_top_fraction(M, w.k)
        sel = zb.zb_block_mass_selected_fraction(M, layer.idx[:1].contiguous())
        torch.cuda.synchronize()
        zb.zb_last_device_status()
        out[name] = {"stage_ms": a.elapsed_time(b) / 3, "retained_mass_top_k_tiles": float(top.mean()),
                     "retained_mass_method_selection": float(sel.mean())}
    out["note"] = ("retained mass: mean over query tiles of head 0 of the dense-softmax mass in the kept key "
                   "tiles; the window stage time includes the three gathers in and the one out")
    del plain, spat, Q, K, V
    torch.cuda.empty_cache()
    return out


def config_dict(w):
    return {"workload": f"{w.name}: {w.n_tokens // synth.TOKENS_PER_VIEW} views x {synth.TOKENS_PER_VIEW} "
                        f"tokens = {w.n_tokens} tokens, {w.heads} heads, d={w.head_dim}, bf16; tile "
                        f"{w.tile}, keep {w.k}/{w.n_tiles} key tiles + landmarks; linear elu+1 with affine "
                        f"fit on {len(synth.calibration_tiles(w.n_tiles, w.calib_tiles)) * w.tile} rows; "
                        f"0.5L/0.5S hybrid",
            "heads": w.heads, "n_tokens": w.n_tokens, "head_dim": w.head_dim, "tile": w.tile, "k": w.k,
            "linear_fraction": 0.5, "l2": l2_note(w.heads * w.n_tokens * w.head_dim * 2)}


L2_BYTES = 126e6


def l2_note(tensor_bytes: float) -> str:
    size = f"each of Q, K, V, O is {tensor_bytes / 1e9:.2f} GB"
    if tensor_bytes > L2_BYTES:
        return f"inputs larger than L2 ({size})"
    return f"inputs smaller than L2 ({size}; the four together {4 * tensor_bytes / 1e9:.2f} GB)"


def main():
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="views1024", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--keep-frac", type=float, default=None, help="override the kept fraction of key tiles")
    ap.add_argument("--heads", type=int, default=None,
                    help="override the head count (a reduced case at full length, for profilers)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-dense-ref", action="store_true", help="skip the dense-attention comparator")
    ap.add_argument("--no-centered", action="store_true", help="skip the linear-centered measurements")
    ap.add_argument("--no-block-mass", action="store_true", help="skip the block-mass diagnostic")
    ap.add_argument("--no-stack", action="store_true", help="skip the 24-layer 512-view stack")
    ap.add_argument("--no-spatial", action="store_true", help="skip the spatial-tiles measurement")
    ap.add_argument("--no-keep20", action="store_true", help="skip the k = ceil(0.2 T) sparse-kernel point")
    ap.add_argument("--profile", action="store_true", help="short run for profilers: no JSON extras")
    args = ap.parse_args()

    w = synth.WORKLOADS[args.workload]
    if args.heads is not None:
        import dataclasses
        w = dataclasses.replace(w, heads=args.heads)
    if args.keep_frac is not None:
        import dataclasses
        w = dataclasses.replace(w, keep_frac=args.keep_frac, k_fixed=None)
    if w.k is None:
        import dataclasses
        w = dataclasses.replace(w, keep_frac=0.06)
    if args.impl == "reference":
        return run_reference(args, w)

    rank, local_rank, world = replicas.env_rank()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (libzb has no CPU path)")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=dev)
    import linear_hybrid_attention_b200 as zb
    zb._lib.load()

    seed = replicas.rank_seed(synth.default_seed(w), rank)
    Q, K, V = synth.make_qkv(w, device=dev, seed=seed)
    calib = synth.calibration_tiles(w.n_tiles, w.calib_tiles)
    layer = zb.HybridLayer(w.heads, w.n_tokens, w.tile, w.k, calib, device=dev)
    stream = torch.cuda.current_stream()

    # per-kernel events around each call of the step (same stream as the kernels)
    names = ["landmark", "topk", "sparse_attn", "linear_state", "calib_dense", "calib_rest", "linear_apply"]

    def run_step(L, q, k, v, ev=None):
        """One pass of the hot path on (q, k, v) with the buffers of HybridLayer L."""
        run_sparse_stage(L, q, k, v, ev)
        run_linear_stage(L, q, k, v, ev)

    def run_sparse_stage(L, q, k, v, ev=None):
        def mark(i):
            if ev is not None:
                ev[i].record(stream)
        mark(0)
        zb.zb_landmark_build(q, k, v, w.tile, out=L.lm)
        mark(1)
        zb.zb_tile_score_topk(L.lm.Qbar, L.lm.Kbar, w.n_tokens, w.tile, w.k, out=L.idx, ws=L.ws_topk)
        mark(2)
        zb.zb_tile_sparse_attn(q, k, v, L.lm.Kbar_bf16, L.lm.Vbar_bf16, L.idx, w.k, w.tile, True,
                               L.scale, out=L.O_sparse, ws=L.ws_attn)
        mark(3)

    def run_linear_stage(L, q, k, v, ev=None):
        def mark(i):
            if ev is not None:
                ev[i].record(stream)
        zb.zb_linear_state(k, v, L.S, L.z, L.ws_lin)
        mark(4)
        zb.zb_gather_tiles(q, w.tile, L.calib, out=L.Qc)
        zb.zb_dense_attn_split(L.Qc, k, v, L.calib_splits, L.scale, out=L.Yc, out_fp32=True, ws=L.ws_dense)
        mark(5)
        zb.zb_linear_apply(L.Qc, L.S, L.z, None, None, out=L.Xc, out_fp32=True)
        zb.zb_affine_fit(L.Xc, L.Yc, L.A, L.b, L.ws_fit)
        mark(6)
        zb.zb_linear_apply(q, L.S, L.z, L.A, L.b, out=L.O_linear)
        mark(7)

    def step(ev=None):
        run_step(layer, Q, K, V, ev)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    zb.zb_last_device_status()
    if args.profile:
        step()
        if not args.no_centered:  # one launch of each linear-centered kernel, for profilers
            mu = zb.zb_key_mean(K)
            zb.zb_linear_state_centered(K, V, mu, ws=layer.ws_lin)
        torch.cuda.synchronize()
        zb.zb_last_device_status()
        if rank == 0:
            print(json.dumps({"profile_run": True, "workload": w.name}))
        return 0

    events = [[torch.cuda.Event(enable_timing=True) for _ in range(8)] for _ in range(args.steps)]
    clocks = ClockSampler(local_rank)
    replicas.barrier(dev)
    torch.cuda.synchronize()
    clocks.start()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for s in range(args.steps):
        step(events[s])
    t_end.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    replicas.barrier(dev)
    zb.zb_last_device_status()
    secs = t_start.elapsed_time(t_end) / 1e3
    tokens_per_step = 2.0 * w.n_tokens  # both stage types of the 0.5L hybrid layer
    tput, t_max = replicas.job_throughput(tokens_per_step, args.steps, secs, dev)
    ms_per_step = t_max / args.steps * 1e3

    per = {n: [] for n in names}
    for ev in events:
        for i, n in enumerate(names):
            per[n].append(ev[i].elapsed_time(ev[i + 1]) / 1e3)
    kt = {n: statistics.median(v) for n, v in per.items()}  # median over the timed steps

    peaks = measured_peaks()
    idx_cpu = layer.idx.cpu().numpy()
    flops = selected_flops(idx_cpu, w.n_tokens, w.tile, w.head_dim)
    sparse_tf = flops / kt["sparse_attn"] / 1e12
    H, N, d = w.heads, w.n_tokens, w.head_dim
    tensor_bytes = H * N * d * 2
    lm_bytes = 3 * tensor_bytes                      # reads Q, K, V once
    lin_state_bytes = 2 * tensor_bytes               # reads K, V
    lin_apply_bytes = 2 * tensor_bytes               # reads Q, writes O
    hbm = peaks["hbm_gbs"]
    traffic, traffic_src = recorded_traffic(w.name)
    roofline = {"kernel": "zb_tile_sparse_attn", "bound": "tensor", "achieved": sparse_tf,
                "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s",
                "frac": sparse_tf / peaks["bf16_tflops_sustained"], "traffic": traffic,
                "traffic_unit": "bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum)",
                "traffic_source": traffic_src,
                "peak_kind": f"bf16 sustained ({peaks['source']}); kernel runs inside a long step",
                "frac_of_burst": sparse_tf / peaks["bf16_tflops"],
                "algorithmic": f"{flops:.4e} FLOP per launch = 4*d*sum n_i*n_j over kept (query tile, key tile) pairs"}
    lm_flops = landmark_flops(w.heads, w.n_tokens, w.n_tiles, w.k, w.head_dim)
    roofline["incl_landmarks"] = {
        "achieved": (flops + lm_flops) / kt["sparse_attn"] / 1e12,
        "frac": (flops + lm_flops) / kt["sparse_attn"] / 1e12 / peaks["bf16_tflops_sustained"],
        "algorithmic": f"{flops + lm_flops:.4e} FLOP per launch: the kept pairs plus 4*d per (query row, landmark) "
                       f"over the T - k landmarks of every row ({lm_flops:.3e})"}
    kernel_rooflines = {
        "zb_landmark_build": {"bound": "hbm", "achieved": lm_bytes / kt["landmark"] / 1e9, "peak": hbm,
                              "unit": "GB/s", "frac": lm_bytes / kt["landmark"] / 1e9 / hbm, "ms": kt["landmark"] * 1e3},
        "zb_linear_state": {"bound": "hbm", "achieved": lin_state_bytes / kt["linear_state"] / 1e9, "peak": hbm,
                            "unit": "GB/s", "frac": lin_state_bytes / kt["linear_state"] / 1e9 / hbm,
                            "ms": kt["linear_state"] * 1e3},
        "zb_linear_apply": {"bound": "hbm", "achieved": lin_apply_bytes / kt["linear_apply"] / 1e9, "peak": hbm,
                            "unit": "GB/s", "frac": lin_apply_bytes / kt["linear_apply"] / 1e9 / hbm,
                            "ms": kt["linear_apply"] * 1e3},
        "zb_linear_attn (state + apply)": {
            "bound": "hbm", "achieved": (lin_state_bytes + lin_apply_bytes) / (kt["linear_state"] + kt["linear_apply"]) / 1e9,
            "peak": hbm, "unit": "GB/s",
            "frac": (lin_state_bytes + lin_apply_bytes) / (kt["linear_state"] + kt["linear_apply"]) / 1e9 / hbm},
        "zb_tile_score_topk": {"ms": kt["topk"] * 1e3, "bound": "hbm (fp32 scores written and read) + alu (select)", "note": "reported only"},
        "calibration (dense 4,096 rows + fit)": {"ms": (kt["calib_dense"] + kt["calib_rest"]) * 1e3},
    }
    stage_ms = {"sparse_stage": (kt["landmark"] + kt["topk"] + kt["sparse_attn"]) * 1e3,
                "linear_stage": (kt["linear_state"] + kt["calib_dense"] + kt["calib_rest"] + kt["linear_apply"]) * 1e3,
                "linear_stage_without_fit": (kt["linear_state"] + kt["linear_apply"]) * 1e3}
    # the pages' headline allocation 0.7L: tokens / (0.7 t_linear + 0.3 t_sparse)
    t_lin = stage_ms["linear_stage"] / 1e3
    t_sp = stage_ms["sparse_stage"] / 1e3
    hybrid_07 = w.n_tokens / (0.7 * t_lin + 0.3 * t_sp) / 1e6 * world

    # --------------------------------------------------- dense comparator ----
    # Dense softmax attention at the same shape, timed on one head (the heads
    # are independent launches of identical cost) and scaled to all heads.
    dense_ref = None
    if not args.no_dense_ref:
        Od = torch.empty((1, w.n_tokens, w.head_dim), dtype=torch.bfloat16, device=dev)
        q1, k1, v1 = Q[:1], K[:1], V[:1]
        zb.zb_dense_attn(q1, k1, v1, layer.scale, out=Od)
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        bb = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        zb.zb_dense_attn(q1, k1, v1, layer.scale, out=Od)
        bb.record(stream)
        torch.cuda.synchronize()
        zb.zb_last_device_status()
        t_head = a.elapsed_time(bb) / 1e3
        dense_flops = 4.0 * w.n_tokens * w.n_tokens * w.head_dim
        dense_ref = {"ms_all_heads": t_head * w.heads * 1e3, "ms_one_head": t_head * 1e3,
                     "tflops": dense_flops / t_head / 1e12,
                     "frac_of_sustained": dense_flops / t_head / 1e12 / peaks["bf16_tflops_sustained"],
                     "sparse_stage_speedup": t_head * w.heads / t_sp,
                     "note": "zb_dense_attn on head 0 at full length, scaled by the head count"}
        del Od

    # ------------------------------------------ the pages' keep-20% point ----
    # The same inputs with k = ceil(0.2 T) (the "0.8S" sparsity of Table 20's
    # allocations): selection, then the tile-sparse kernel timed on its own
    # (one warm-up launch, two timed), against the same sustained peak.
    keep20 = None
    if not args.no_keep20 and w.name == "views1024":
        k20 = -(-w.n_tiles // 5)
        idx20 = torch.empty((w.heads, w.n_tiles, k20), dtype=torch.int32, device=dev)
        zb.zb_tile_score_topk(layer.lm.Qbar, layer.lm.Kbar, w.n_tokens, w.tile, k20, out=idx20, ws=layer.ws_topk)
        n_t = torch.full((w.n_tiles,), float(w.tile), dtype=torch.float64, device=dev)
        n_t[-1] = w.n_tokens - (w.n_tiles - 1) * w.tile
        fl20 = sum(float(4.0 * w.head_dim * (n_t[idx20[h].long()].sum(-1) * n_t).sum().item())
                   for h in range(w.heads))
        lm20 = landmark_flops(w.heads, w.n_tokens, w.n_tiles, k20, w.head_dim)
        run20 = lambda: zb.zb_tile_sparse_attn(Q, K, V, layer.lm.Kbar_bf16, layer.lm.Vbar_bf16, idx20, k20, w.tile,
                                               True, layer.scale, out=layer.O_sparse, ws=layer.ws_attn)
        run20()
        torch.cuda.synchronize()
        e20 = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        e20[0].record(stream)
        run20()
        e20[1].record(stream)
        run20()
        e20[2].record(stream)
        torch.cuda.synchronize()
        zb.zb_last_device_status()
        t20 = statistics.mean([e20[0].elapsed_time(e20[1]), e20[1].elapsed_time(e20[2])]) / 1e3
        keep20 = {"k": k20, "ms": t20 * 1e3, "tflops": fl20 / t20 / 1e12,
                  "frac": fl20 / t20 / 1e12 / peaks["bf16_tflops_sustained"],
                  "frac_incl_landmarks": (fl20 + lm20) / t20 / 1e12 / peaks["bf16_tflops_sustained"],
                  "note": "zb_tile_sparse_attn alone on the 1,024-view inputs with the k = ceil(0.2 T) selection; "
                          "frac on selected-tile FLOPs against the sustained bf16 peak"}
        del idx20

    # -------------------------------------------- linear-centered variant ----
    # Outside the timed step: the centred linear stage (keys shifted by their
    # per-head mean) on the same inputs, its two new kernels against HBM, and
    # the fitted output's residual against dense attention with and without
    # centring, on the calibration rows and on as many held-out rows.
    centered = None
    if not args.no_centered:
        centered = linear_centered_report(zb, w, layer, Q, K, V, stream, hbm, tensor_bytes, kt["linear_apply"])

    # --------------------------------------------- block-mass diagnostic ----
    block_mass = None
    if not args.no_block_mass:
        block_mass = block_mass_report(zb, w, layer, Q, K, V, stream)

    # ------------------------------------------------------------ e2e ----
    # The same steps through the public calls with the inputs copied in from
    # pinned host memory and both outputs copied back, every step, inside the
    # timed region: once serially on the compute stream, and once pipelined
    # (step s + 1's inputs copied in and step s - 1's outputs copied out on two
    # copy streams while step s computes; two buffer sets alternate).
    e2e = None
    if not args.no_e2e:
        pin = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in (Q, K, V)]
        outs = [torch.empty(Q.shape, dtype=Q.dtype, pin_memory=True) for _ in range(2)]
        for p_, t in zip(pin, (Q, K, V)):
            p_.copy_(t)
        e2e_steps = 8  # the pipeline fill and drain amortised over 8 steps whatever --steps is

        def e2e_step():
            for p_, t in zip(pin, (Q, K, V)):
                t.copy_(p_, non_blocking=True)
            step()
            outs[0].copy_(layer.O_sparse, non_blocking=True)
            outs[1].copy_(layer.O_linear, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        replicas.barrier(dev)
        a = torch.cuda.Event(enable_timing=True)
        bb = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        bb.record(stream)
        torch.cuda.synchronize()
        replicas.barrier(dev)
        serial_secs = a.elapsed_time(bb) / 1e3
        serial_tput, _ = replicas.job_throughput(tokens_per_step, e2e_steps, serial_secs, dev)

        # pipelined
        layer2 = zb.HybridLayer(w.heads, w.n_tokens, w.tile, w.k, calib, device=dev)
        layers = [layer, layer2]
        din = [(Q, K, V), tuple(torch.empty_like(t) for t in (Q, K, V))]
        cin, cout = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

        def pipelined(n):
            in_ready = [torch.cuda.Event() for _ in range(n)]
            lin_done = [torch.cuda.Event() for _ in range(n)]
            done = [torch.cuda.Event() for _ in range(n)]
            out_done = [torch.cuda.Event() for _ in range(n)]
            cin.wait_stream(stream)
            with torch.cuda.stream(cin):
                for p_, t in zip(pin, din[0]):
                    t.copy_(p_, non_blocking=True)
                in_ready[0].record(cin)
            for s_ in range(n):
                b_ = s_ % 2
                if s_ + 1 < n:
                    if s_ >= 1:
                        cin.wait_event(done[s_ - 1])          # step s - 1 has read din[(s + 1) % 2]
                    with torch.cuda.stream(cin):
                        for p_, t in zip(pin, din[(s_ + 1) % 2]):
                            t.copy_(p_, non_blocking=True)
                        in_ready[s_ + 1].record(cin)
                stream.wait_event(in_ready[s_])
                if s_ >= 2:
                    stream.wait_event(out_done[s_ - 2])        # layers[b]'s outputs are out
                # the linear stage first, so that its output moves out while the
                # sparse stage computes and only the sparse output is left to drain
                run_linear_stage(layers[b_], *din[b_])
                lin_done[s_].record(stream)
                cout.wait_event(lin_done[s_])
                with torch.cuda.stream(cout):
                    outs[1].copy_(layers[b_].O_linear, non_blocking=True)
                run_sparse_stage(layers[b_], *din[b_])
                done[s_].record(stream)
                cout.wait_event(done[s_])
                with torch.cuda.stream(cout):
                    outs[0].copy_(layers[b_].O_sparse, non_blocking=True)
                    out_done[s_].record(cout)
            stream.wait_event(out_done[n - 1])

        pipelined(2)
        torch.cuda.synchronize()
        replicas.barrier(dev)
        a.record(stream)
        pipelined(e2e_steps)
        bb.record(stream)
        torch.cuda.synchronize()
        replicas.barrier(dev)
        zb.zb_last_device_status()
        e_secs = a.elapsed_time(bb) / 1e3
        e_tput, _ = replicas.job_throughput(tokens_per_step, e2e_steps, e_secs, dev)
        e2e = {"value": e_tput / 1e6, "unit": UNIT, "h2d_bytes_per_step": 3 * tensor_bytes,
               "d2h_bytes_per_step": 2 * tensor_bytes, "steps": e2e_steps,
               "api": "HybridLayer C-ABI calls; every step's Q, K, V copied in from pinned host memory and both "
                      "outputs copied back inside the timed region, pipelined: the next step's inputs and the "
                      "previous step's outputs move on two copy streams while a step computes (each step runs "
                      "its linear stage first, whose output then moves out during the sparse stage)",
               "serial_value": serial_tput / 1e6,
               "serial_note": "the same with every copy on the compute stream, no overlap"}
        del pin, outs, layer2, layers, din

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        t_cpu, desc, cores = oracle_sample(w, Q, K, V, calib)
        cpu = {"value": tokens_per_step / t_cpu / 1e6, "unit": UNIT, "cores": cores, "cpu_model": cpu_model(),
               "kind": "oracle",
               "sample": desc}

    # read-only HBM stream rate (a second denominator for the HBM-bound kernels)
    read_gbs = read_stream_gbs(dev)
    for kr in kernel_rooflines.values():
        if kr.get("bound") == "hbm":
            kr["frac_of_read_stream"] = kr["achieved"] / read_gbs
            kr["frac_of_spec"] = kr["achieved"] / SPEC_HBM_GBS
    if centered is not None:
        for kr in (centered["zb_key_mean"], centered["zb_linear_state_centered"]):
            kr["frac_of_read_stream"] = kr["achieved"] / read_gbs
            kr["frac_of_spec"] = kr["achieved"] / SPEC_HBM_GBS
    hbm_peaks = {"copy_gbs (MEASURED_PEAKS.json, the roofline peak)": hbm, "read_stream_gbs (measured here)": read_gbs,
                 "spec_gbs": SPEC_HBM_GBS}
    # the same kernels alone, at the clock they then run at: the in-step figures
    # above run at the clock the long tile-sparse kernel leaves under the power cap
    iso = hbm_isolated({
        "zb_landmark_build": lambda: zb.zb_landmark_build(Q, K, V, w.tile, out=layer.lm),
        "zb_linear_state": lambda: zb.zb_linear_state(K, V, layer.S, layer.z, layer.ws_lin),
        "zb_linear_apply": lambda: zb.zb_linear_apply(Q, layer.S, layer.z, layer.A, layer.b, out=layer.O_linear),
    }, dev, local_rank)
    iso_bytes = {"zb_landmark_build": lm_bytes, "zb_linear_state": lin_state_bytes, "zb_linear_apply": lin_apply_bytes}
    for n, ms in iso["ms"].items():
        kernel_rooflines[n]["alone"] = {"ms": ms, "frac": iso_bytes[n] / (ms / 1e3) / 1e9 / hbm}
    t_iso = iso["ms"]["zb_linear_state"] + iso["ms"]["zb_linear_apply"]
    kernel_rooflines["zb_linear_attn (state + apply)"]["alone"] = {
        "ms": t_iso, "frac": (lin_state_bytes + lin_apply_bytes) / (t_iso / 1e3) / 1e9 / hbm}
    hbm_clocks = {"in_step": clk, "alone": iso["clocks"],
                  "note": "frac is measured inside the timed step (clocks: the step's samples, mostly during the "
                          "tile-sparse kernel); alone = each kernel launched back to back for 0.5 s with L2 "
                          "flushed before every launch (clocks sampled over that loop)"}

    # the step without calibration: the affine fit done once, offline, and the
    # fitted (A, b) reused -- the linear stage is then its two passes
    t_offline = kt["landmark"] + kt["topk"] + kt["sparse_attn"] + kt["linear_state"] + kt["linear_apply"]
    value_fit_offline = tokens_per_step / t_offline / 1e6 * world

    gpu_launches = layer.launches_per_step * args.steps
    spatial = None
    if not args.no_spatial and w.name == "views1024":
        spatial = spatial_report(zb, dev, stream)
    stack = None
    if not args.no_stack and w.name == "views1024":
        del Q, K, V, layer
        torch.cuda.empty_cache()
        stack = stack_report(zb, rank, dev, stream)

    if rank == 0:
        line = {"metric": METRIC, "value": tput / 1e6, "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": config_dict(w), "e2e": e2e, "gpu_launches": gpu_launches,
                "roofline": roofline, "kernel_roofline": kernel_rooflines, "stage_ms": stage_ms,
                "kernel_ms": {n: v * 1e3 for n, v in kt.items()}, "clocks": clk, "cpu_baseline": cpu,
                "hybrid_0.7L_mtokens_s": hybrid_07, "dense_reference": dense_ref, "linear_centered": centered,
                "block_mass": block_mass, "stack512": stack, "spatial_tiles": spatial, "keep20": keep20,
                "value_definition": "value = 2 N / t_step with every call of the hot path in the step, the "
                                    "calibration (dense attention on 4,096 rows) and the affine fit included",
                "value_fit_offline": value_fit_offline,
                "value_fit_offline_definition": "2 N / (landmarks + selection + tile-sparse attention + linear "
                                                "state + fitted linear output): the fit done once, offline",
                "hbm_peaks": hbm_peaks, "hbm_kernel_clocks": hbm_clocks, "peaks": peaks}
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
