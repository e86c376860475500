"""Benchmark of one DSpark draft/verify round on B200 (one JSON line on rank 0).

Default workload (the headline): high concurrency, B=64 requests, gamma=16, V=151936, r=256,
T=0.8, bf16 Markov-head weights, fp32 logits (synthetic, seeded; see inputs.py).  --workload
selects another of the five cases: single_user (B=1, gamma=7, T=1), single_user_greedy (T=0),
scheduled_step (B=256, gamma=5, V=129280, the scheduler's verify lengths), sweep_B{B}_g{gamma}
(V=262144, B in 1/8/32/128/512, gamma in 4/8/16), or profile (B=64, gamma=4: the headline's kernels
on about 0.6 GB, for ncu captures).

One step = one pass of the whole hot path over one batch:
  markov_draft (gamma positions in one cooperative launch on the tensor-core path)
  -> prefix_schedule (prefix survival + greedy scheduler; a flat steps/s table, so the whole
     gamma-block is verified, except on scheduled_step, which uses its affine-latency table)
  -> verify (acceptance, residual/bonus sample; TV labels fused in, except on scheduled_step,
     where only the scheduled rows are read).
Inputs live in HBM when the timed region starts; L2 (126 MB) is flushed by writing a 256 MB
buffer before every timed step, outside the timed events ("warm" repeats the timing without it).
Times are medians of the per-step CUDA-event times on the launching stream.

value       = rounds/s over all ranks (each rank runs its own batch: weak scaling)
e2e         = the same rounds/s through the public API with pinned host buffers: the per-step
              inputs are copied host->device and the step's result (n_acc, y) device->host
              inside the timed region
roofline    = the draft stage (its one launch) against measured HBM copy bandwidth, algorithmic
              bytes B*gamma*V*4 (read U) + gamma*r*V*2 (W2 per position) + B*gamma*V*4 (write l_d);
              the verify call is reported beside it (rows it must read: every l_d and l_t row
              with labels, else the scheduled ones)
cpu_baseline= the CPU oracle on the machine's host cores: its request-independent and per-request
              costs timed separately on small samples and combined for the whole batch

graph_t2    = the round captured once as a CUDA graph with the asynchronous (t-2) scheduler and
              replayed, L2 flushed between replays

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--workload NAME]
                  [--layout position|request] [--labels auto|on|off]
  python bench.py --draft-crossover     # draft time on the GEMV and tensor-core paths over B
  python bench.py --calibration         # sequential temperature scaling: fit and apply timings
"""

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "draft+verify rounds/s and verified tokens/s at V=151936, γ=16; HBM GB/s vs peak"
UNIT = "rounds/s"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
HOST_E2E_LIMIT = 6 << 30   # larger per-step inputs (big sweep points) are not staged in pinned memory


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), float(j.get("bf16_tflops", FALLBACK_BF16_TFLOPS)), "measured"
    return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


def measured_traffic(key, units):
    """DRAM bytes (read + write) of one launch of kernel `key` from the ncu capture summarised in
    profiles/traffic.json, scaled to `units` of work; None when that kernel's source file has
    changed since the counters were taken (its SHA-1 is stored beside them)."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            t = json.load(f)[key]
        with open(os.path.join(ROOT, "speculative_decoding_04_b200", "csrc", t["source"]), "rb") as f:
            sha = hashlib.sha1(f.read()).hexdigest()
    except (OSError, KeyError, ValueError):
        return None
    if sha != t.get("source_sha1"):
        return None
    return t["dram_bytes_per_launch"] * units / t["units_per_launch"]


def workload_of(name):
    from speculative_decoding_04_b200 import inputs

    if name in inputs.WORKLOADS:
        return inputs.WORKLOADS[name]
    if name == "profile":
        return inputs.HIGH_CONCURRENCY.with_(name="profile", B=64, gamma=4)
    if name.startswith("sweep_B"):
        b, g = name[len("sweep_B"):].split("_g")
        return inputs.sweep_point(int(b), int(g))
    raise SystemExit(f"unknown workload {name}")


def uses_schedule_table(wl):
    return wl.name == "scheduled_step"


def draft_bytes(wl):
    B, G, V, r = wl.B, wl.gamma, wl.V, wl.r
    return B * G * V * 4 + G * r * V * 2 + B * G * V * 4


def verify_bytes(wl, L=None, labels=True):
    """Rows the verification must read: every l_d and l_t row with labels; else l_d rows
    k < L_b and l_t rows k <= L_b of each request."""
    B, G, V = wl.B, wl.gamma, wl.V
    if labels or L is None:
        return B * G * V * 4 + B * (G + 1) * V * 4
    L = np.asarray(L, dtype=np.int64)
    return int((2 * L + 1).sum()) * V * 4


def config_of(wl, n, labels, layout="position", ragged=False):
    return {"layout": ("position-major [gamma, B, V]" if layout == "position" else "request-major [B, gamma, V]")
                      + " draft logits U and ld",
            "lt_layout": "flattened [sum(L_b + 1), V] with row offsets" if ragged else "padded [B, gamma + 1, V]",
            "workload": f"{wl.name}: B={wl.B} requests, gamma={wl.gamma}, V={wl.V}, r={wl.r}, T={wl.T}, "
                        f"{wl.w_dtype} W1/W2, fp32 {'log-Zipf+Gaussian' if wl.logits == 'logzipf' else 'Gaussian'} "
                        "logits",
            "B_per_gpu": wl.B, "gamma": wl.gamma, "V": wl.V, "r": wl.r, "T": wl.T,
            "parallelism": f"replicas over {n} GPU(s), no data-path collective",
            "l2_policy": "256 MB write before every timed step (outside the timed events); inputs > L2 too",
            "step": ("markov_draft -> prefix_schedule ("
                     + ("affine-latency sps, scheduled lengths" if uses_schedule_table(wl) else "flat sps, full block")
                     + ") -> verify" + (" (+TV labels)" if labels else " (scheduled rows only)"))}


class Clocks:
    """nvidia-smi sampled during the timed region; the raw samples go to clocks_<gpu>.csv in the
    directory named by DSPARK_CLOCKS_DIR (default: the system temporary directory)."""

    def __init__(self, index):
        self.path = os.path.join(os.environ.get("DSPARK_CLOCKS_DIR", tempfile.gettempdir()), f"clocks_{index}.csv")
        os.makedirs(os.path.dirname(self.path), exist_ok=True)
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.f = open(self.path, "w")
            self.p = subprocess.Popen(["nvidia-smi", "-i", str(index), f"--query-gpu={q}", "--format=csv,noheader",
                                       "-lms", "100"], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.p = None

    def stop(self):
        if self.p is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.p.terminate()
        self.p.wait()
        self.f.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1].split()[0]))
                smax.append(float(f[2].split()[0]))
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def oracle_round(wl, reqs, labels):
    """One full oracle round (draft, schedule, verify, labels) on the given requests; seconds."""
    import oracle as O
    from speculative_decoding_04_b200 import inputs

    U, lt = inputs.logits(wl, reqs)
    W1, W2 = inputs.weights(wl)
    x0 = inputs.tokens(wl)[reqs]
    u_draft, u_acc, u_res = (a[reqs] for a in inputs.uniforms(wl))
    c = inputs.confidences(wl)
    sps = inputs.sps_table(wl) if uses_schedule_table(wl) else np.ones(wl.D_max + 1)
    t0 = time.perf_counter()
    x, ld, _ = O.markov_draft(U, W1, W2, x0, u_draft, wl.T)
    sch = O.prefix_schedule(c, sps, wl.D_max)
    O.verify(ld, lt, x, sch["L"][reqs], u_acc, u_res, wl.T)
    if labels:
        O.tv_labels(ld, lt[:, :wl.gamma], wl.T)
    return time.perf_counter() - t0


def cpu_baseline(wl, labels, n1=1, n2=3):
    """The oracle (as it stands) on the host cores.  A round's cost is a request-independent part
    (the fp64 copy of W2, the scheduler over the whole batch) plus a per-request part; both come
    from timing one round on n1 and on n2 requests, and are combined for the whole batch."""
    threads = os.cpu_count() or 1
    n1, n2 = min(n1, wl.B), min(n2, wl.B)
    t1 = oracle_round(wl, list(range(n1)), labels)
    if n2 <= n1:  # the whole batch is the sample
        return {"value": 1.0 / t1, "unit": UNIT, "cores": threads, "kind": "oracle",
                "sample": f"one round on all {wl.B} request(s), {t1:.2f} s"}
    t2 = oracle_round(wl, list(range(n2)), labels)
    per_req = max((t2 - t1) / (n2 - n1), 1e-9)
    fixed = max(t1 - n1 * per_req, 0.0)
    per_round = fixed + wl.B * per_req
    return {"value": 1.0 / per_round, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"one round on {n1} and on {n2} of {wl.B} requests ({t1:.2f} s, {t2:.2f} s): "
                      f"{fixed:.2f} s request-independent + {per_req:.2f} s per request, "
                      f"= {per_round:.1f} s for the whole batch"}


def rank_workload(wl, rank):
    """Each rank verifies its own batch of B requests (weak scaling): rank r > 0 shifts the seed."""
    return wl.with_(seed=wl.seed + 1000 * rank) if rank else wl


def combine_ranks(times, accepted, world, device):
    """Device times: the max over ranks of each; accepted tokens: the sum over ranks."""
    import torch
    import torch.distributed as dist

    vals = torch.tensor(list(times), dtype=torch.float64, device=device)
    tot = torch.tensor([float(accepted)], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(vals, op=dist.ReduceOp.MAX)
        dist.all_reduce(tot, op=dist.ReduceOp.SUM)
    return vals.tolist(), tot.item()


def run_reference(args, wl, labels, rank):
    """The reference arm: the CPU oracle as it stands.  Each step is one oracle round on a
    bounded sample of requests (n_req of B); rounds/s of the whole batch come from the sample's
    request-independent and per-request costs (timed once, as cpu_baseline does)."""
    if rank != 0:
        return
    n_req = 1
    cb = cpu_baseline(wl, labels)
    steps = []
    for i in range(args.warmup + args.steps):
        t = oracle_round(wl, list(range(n_req)), labels)
        if i >= args.warmup:
            steps.append(t)
    t_step = statistics.median(steps)
    line = {"impl": "reference", "metric": METRIC, "value": cb["value"], "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_step * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded, see inputs.py)",
            "config": config_of(wl, args.gpus, labels, args.layout, args.ragged),
            "cpu_baseline": dict(cb, sample=cb["sample"] + f"; each timed step: one round on {n_req} request(s)"),
            "e2e": {"value": cb["value"], "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)


def median_ms(pairs):
    return statistics.median(a.elapsed_time(b) for a, b in pairs)


def draft_crossover(args):
    """Draft time (CUDA events, median of 10 after 3 warm-ups, L2 flushed) on the CUDA-core GEMV
    path and on the tensor-core path for B = 1 .. 32 at gamma = 16, V = 151936, r = 256."""
    import torch

    from speculative_decoding_04_b200 import build
    build.build()
    from speculative_decoding_04_b200 import dspark as D
    from speculative_decoding_04_b200 import inputs

    dev = torch.device("cuda")
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    base = inputs.HIGH_CONCURRENCY
    W1h, W2h = inputs.weights(base)
    W1 = torch.from_numpy(W1h).to(torch.bfloat16).to(dev)
    W2 = torch.from_numpy(W2h).to(torch.bfloat16).to(dev)
    for B in (1, 2, 4, 8, 9, 12, 16, 24, 32):
        wl = base.with_(B=B)
        U, _ = inputs.device_logits(wl, dev)
        x0 = torch.from_numpy(inputs.tokens(wl)).to(dev)
        u = torch.from_numpy(inputs.uniforms(wl)[0]).to(dev)
        row = {"B": B, "gamma": wl.gamma, "V": wl.V}
        for path, name in ((1, "gemv_ms"), (2, "tensor_core_ms")):
            D.set_option("draft_path", path)
            ev = []
            for i in range(13):
                flush.fill_(float(i))
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                D.markov_draft(U, W1, W2, x0, u, wl.T)
                e1.record()
                if i >= 3:
                    ev.append((e0, e1))
            torch.cuda.synchronize()
            row[name] = median_ms(ev)
        D.set_option("draft_path", 0)
        row["draft_bytes_GB"] = draft_bytes(wl) / 1e9
        print(json.dumps(row), flush=True)
        del U
        torch.cuda.empty_cache()


def calibration(args):
    """Sequential temperature scaling: sts_fit on a validation set of N = 1,000,000 samples, gamma = 16,
    81 grid temperatures, 15 bins (CUDA events, median of --steps after --warmup), the oracle's
    sts_fit on a 20,000-sample slice of it (one run), and sts_apply on the high-concurrency
    round's [64, 16] confidences."""
    import torch

    from speculative_decoding_04_b200 import build
    build.build()
    from speculative_decoding_04_b200 import dspark as D
    from speculative_decoding_04_b200 import inputs

    dev = torch.device("cuda")
    N, G, M = 1_000_000, 16, 15
    grid_h = np.exp(np.linspace(np.log(0.25), np.log(4.0), 81))
    c_h, n_h = inputs.calibration_set(N, G, seed=11)
    c, n, grid = (torch.from_numpy(v).to(dev) for v in (c_h, n_h, grid_h))
    ws = torch.empty(D.lib.dspark_sts_workspace_size(N, G, grid.numel(), M), dtype=torch.uint8, device=dev)
    ev = []
    for i in range(args.warmup + args.steps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        out = D.sts_fit(c, n, grid, M, ws=ws)
        e1.record()
        if i >= args.warmup:
            ev.append((e0, e1))
    torch.cuda.synchronize()
    fit_ms = median_ms(ev)
    evals = N * G * (grid.numel() + 1)
    rc = inputs.confidences(inputs.HIGH_CONCURRENCY)
    rcd = torch.from_numpy(rc).to(dev)
    ev = []
    for i in range(args.warmup + args.steps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        D.sts_apply(rcd, out["tau"])
        e1.record()
        if i >= args.warmup:
            ev.append((e0, e1))
    torch.cuda.synchronize()
    apply_ms = median_ms(ev)
    import oracle as O
    cpu_n = 20_000
    t0 = time.perf_counter()
    O.sts_fit(c_h[:cpu_n], n_h[:cpu_n], grid_h, M)
    cpu_s = time.perf_counter() - t0
    line = {"metric": "sts_fit (sample, position, temperature) evaluations/s", "value": evals / (fit_ms * 1e-3),
            "unit": "evaluations/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": fit_ms,
            "higher_is_better": True, "dtype": "f64", "data": "synthetic (inputs.calibration_set)",
            "config": {"workload": f"validation set N={N}, gamma={G}, {grid.numel()} grid temperatures, {M} bins"},
            "ece_raw_pct": [round(100 * v, 3) for v in out["ece_raw"].tolist()],
            "ece_cal_pct": [round(100 * v, 3) for v in out["ece_cal"].tolist()],
            "tau": [round(v, 4) for v in out["tau"].tolist()],
            "sts_apply_us": apply_ms * 1e3, "gpu_launches": 2 * G + 1,
            "cpu_baseline": {"value": cpu_n * G * (grid.numel() + 1) / cpu_s, "unit": "evaluations/s", "cores": 1,
                             "kind": "oracle", "sample": f"oracle sts_fit on the first {cpu_n} samples, one run"}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="dspark", choices=["dspark", "reference"])
    ap.add_argument("--workload", default="high_concurrency",
                    help="high_concurrency (default), single_user, single_user_greedy, scheduled_step, "
                         "sweep_B{B}_g{gamma}, profile")
    ap.add_argument("--labels", choices=["auto", "on", "off"], default="auto",
                    help="TV labels in the verify call (auto: on, except on scheduled_step)")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the CPU oracle timing (after the GPU timing)")
    ap.add_argument("--draft-crossover", action="store_true", help="print draft times of both main-pass paths over B")
    ap.add_argument("--ragged", action="store_true",
                    help="target logits as a flattened block of the scheduled rows (sum of L_b + 1 rows) and the "
                         "flattened verify")
    ap.add_argument("--calibration", action="store_true",
                    help="time sequential temperature scaling (sts_fit, sts_apply) instead of the round")
    ap.add_argument("--layout", choices=["position", "request"], default="position",
                    help="layout of the draft logits U and of ld: position-major [gamma, B, V] (default) or "
                         "request-major [B, gamma, V]")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.draft_crossover:
        return draft_crossover(args)
    if args.calibration:
        return calibration(args)

    wl = workload_of(args.workload)
    labels = (args.labels == "on") or (args.labels == "auto" and not uses_schedule_table(wl))
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if args.impl == "reference":
        return run_reference(args, wl, labels, rank)

    import torch
    import torch.distributed as dist

    from speculative_decoding_04_b200 import build
    build.build()
    from speculative_decoding_04_b200 import dspark as D
    from speculative_decoding_04_b200 import inputs

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    # ---------------------------------------------------------------- inputs (each rank its own batch)
    wr = rank_workload(wl, rank)
    B, G, V, r = wl.B, wl.gamma, wl.V, wl.r
    wdt = torch.bfloat16 if wl.w_dtype == "bf16" else torch.float32
    W1h, W2h = inputs.weights(wr)
    W1 = torch.from_numpy(W1h).to(wdt).to(dev)
    W2 = torch.from_numpy(W2h).to(wdt).to(dev)
    u_draft, u_acc, u_res = inputs.uniforms(wr)
    small = {"x0": inputs.tokens(wr), "u_draft": u_draft, "u_acc": u_acc, "u_res": u_res, "c": inputs.confidences(wr)}
    dv = {k: torch.from_numpy(np.ascontiguousarray(v)).to(dev) for k, v in small.items()}
    host_logit_bytes = (B * G * V + B * (G + 1) * V) * 4
    if wl.name.startswith("sweep_B"):
        dv["U"], dv["lt"] = inputs.device_logits(wr, dev)          # drawn on the device (up to 26 GB)
        if args.layout == "request":
            dv["U"] = dv["U"].transpose(0, 1).contiguous()
    else:
        U, lt = inputs.logits(wr)
        Uh = U.transpose(1, 0, 2) if args.layout == "position" else U
        dv["U"] = torch.from_numpy(np.ascontiguousarray(Uh)).to(dev)
        dv["lt"] = torch.from_numpy(lt).to(dev)
        del U, lt, Uh
    sps_h = inputs.sps_table(wr) if uses_schedule_table(wl) else np.ones(B * G + 1)
    sps = torch.from_numpy(sps_h).to(dev)
    lt_off = None
    if args.ragged:
        # the target block as a target forward over the scheduled tokens would emit it: rows
        # 0..L_b of each request, flattened (the schedule is deterministic for these inputs)
        L0 = torch.empty(B, dtype=torch.int32, device=dev)
        D.prefix_schedule(dv["c"], sps, B * G, L_out=L0, want_a=False)
        L0h = L0.cpu().numpy()
        rows = np.concatenate([b * (G + 1) + np.arange(int(l) + 1) for b, l in enumerate(L0h)])
        dv["lt"] = dv["lt"].view(B * (G + 1), V).index_select(0, torch.from_numpy(rows).to(dev)).contiguous()
        host_logit_bytes = (B * G * V + dv["lt"].shape[0] * V) * 4
        lt_off = torch.empty(B + 1, dtype=torch.int64, device=dev)
        torch.cuda.synchronize(dev)
    x = torch.empty((B, G), dtype=torch.int32, device=dev)
    ld = torch.empty(tuple(dv["U"].shape), dtype=torch.float32, device=dev)
    fl = torch.zeros(B, dtype=torch.int32, device=dev)
    L = torch.empty(B, dtype=torch.int32, device=dev)
    theta = torch.empty(1, dtype=torch.float64, device=dev)
    n_acc = torch.empty(B, dtype=torch.int32, device=dev)
    y = torch.empty((B, G + 1), dtype=torch.int32, device=dev)
    c_star = torch.empty((B, G), dtype=torch.float32, device=dev) if labels else None
    ws_d = D.workspace(D.WS_DRAFT, B, G, V, r, dev)
    ws_v = D.workspace(D.WS_VERIFY, B, G, V, 0, dev)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(device=dev)
    # draft: one cooperative launch on the tensor-core path, else a main pass and a combine per
    # position; schedule; verify: main kernel + finalize
    tc = wl.w_dtype == "bf16" and r % 64 == 0 and r <= 256 and V % 8 == 0
    n_launch = (1 if tc else 2 * G) + 1 + 2 + (1 if args.ragged else 0)

    def draft(src):
        D.markov_draft(src["U"], W1, W2, src["x0"], src["u_draft"], wl.T, layout=args.layout, x_out=x, ld_out=ld,
                       flags=fl, ws=ws_d, stream=stream)

    def verify_call(src):
        if args.ragged:
            D.ragged_layout(L, G, lt_off=lt_off, want_tags=False, stream=stream)
            D.verify_ragged(ld, src["lt"], lt_off, x, L, src["u_acc"], src["u_res"], wl.T, ld_layout=args.layout,
                            n_acc=n_acc, y_out=y, c_star=c_star, flags=fl, ws=ws_v, stream=stream)
        else:
            D.verify(ld, src["lt"], x, L, src["u_acc"], src["u_res"], wl.T, ld_layout=args.layout, n_acc=n_acc,
                     y_out=y, c_star=c_star, flags=fl, ws=ws_v, stream=stream)

    def schedule_and_verify(src):
        D.prefix_schedule(src["c"], sps, B * G, D.SCHED_ARGMAX, L_out=L, theta_out=theta, flags=fl, want_a=False,
                          stream=stream)
        verify_call(src)

    def barrier():
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    def timed_rounds(nsteps, cold):
        ev = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3)) for _ in range(nsteps)]
        acc_dev = torch.zeros((), dtype=torch.int64, device=dev)
        for i in range(nsteps):
            if cold:
                flush.fill_(float(i))
            ev[i][0].record(stream)
            draft(dv)
            ev[i][1].record(stream)
            schedule_and_verify(dv)
            ev[i][2].record(stream)
            acc_dev += n_acc.sum() + B
        barrier()
        step = statistics.median(a.elapsed_time(c) for a, _, c in ev)
        dr = statistics.median(a.elapsed_time(b) for a, b, _ in ev)
        return step, dr, int(acc_dev.item())

    clk = Clocks(local)      # sampling starts before the warm-up so that it covers the timed region
    time.sleep(0.5)
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            flush.fill_(1.0)
            draft(dv)
            schedule_and_verify(dv)
        barrier()
        tw0 = time.perf_counter()
        step_ms, draft_ms, accepted = timed_rounds(args.steps, cold=True)
        tw1 = time.perf_counter()
        clocks = clk.stop()
        L_h = L.cpu().numpy()
        warm_step_ms, warm_draft_ms, _ = timed_rounds(args.steps, cold=False)

        # verify alone (schedule + verify for the scheduled workload), timed live after a flush
        vt = []
        for i in range(args.steps):
            flush.fill_(float(i))
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            verify_call(dv)
            e1.record(stream)
            vt.append((e0, e1))
        barrier()
        verify_ms = median_ms(vt)

        # back-to-back rounds through the API without flushes or syncs: host wall clock per round
        # against device time (launch overheads of the calls)
        barrier()
        tb0 = time.perf_counter()
        eb0, eb1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        eb0.record(stream)
        for _ in range(args.steps):
            draft(dv)
            schedule_and_verify(dv)
        eb1.record(stream)
        th = time.perf_counter()
        barrier()
        tb1 = time.perf_counter()
        b2b = {"rounds": args.steps, "host_issue_ms_per_round": (th - tb0) * 1e3 / args.steps,
               "wall_ms_per_round": (tb1 - tb0) * 1e3 / args.steps,
               "device_ms_per_round": eb0.elapsed_time(eb1) / args.steps}

        # the round captured once as a CUDA graph and replayed, with the asynchronous scheduler
        # (capacity from step t-2, kept on a device ring), L2 flushed before every replay
        ring = D.schedule_ring(dev)
        K_t = torch.empty(1, dtype=torch.int32, device=dev)

        def round_t2(src):
            draft(src)
            D.prefix_schedule_t2(src["c"], sps, B * G, ring, L_out=L, theta_out=theta, K_out=K_t, flags=fl,
                                 stream=stream)
            D.verify(ld, src["lt"], x, L, src["u_acc"], src["u_res"], wl.T, ld_layout=args.layout, n_acc=n_acc,
                     y_out=y, c_star=c_star, flags=fl, ws=ws_v, stream=stream)

        graph_ms = None
        if not args.ragged:   # (the t-2 schedule's lengths are not the ones the flattened block holds)
            round_t2(dv)
            barrier()
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, stream=stream):
                round_t2(dv)
            gt = []
            for i in range(args.warmup + args.steps):
                flush.fill_(float(i))
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                graph.replay()
                e1.record(stream)
                if i >= args.warmup:
                    gt.append((e0, e1))
            barrier()
            graph_ms = median_ms(gt)
            del graph

        # end to end through the public API with pinned host buffers
        e2e = None
        if host_logit_bytes <= HOST_E2E_LIMIT:
            pin = {k: torch.empty(v.shape, dtype=v.dtype).pin_memory() for k, v in dv.items()}
            for k in pin:
                pin[k].copy_(dv[k])
            n_out = torch.empty(B, dtype=torch.int32).pin_memory()
            y_out = torch.empty((B, G + 1), dtype=torch.int32).pin_memory()
            h2d = sum(v.numel() * v.element_size() for v in pin.values())
            d2h = n_out.numel() * 4 + y_out.numel() * 4
            stage = {k: torch.empty_like(v) for k, v in dv.items()}
            ev = []
            for i in range(args.warmup + args.steps):
                flush.fill_(float(i))
                barrier()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                for k in stage:
                    stage[k].copy_(pin[k], non_blocking=True)
                draft(stage)
                schedule_and_verify(stage)
                n_out.copy_(n_acc, non_blocking=True)
                y_out.copy_(y, non_blocking=True)
                e1.record(stream)
                e1.synchronize()
                if i >= args.warmup:
                    ev.append((e0, e1))
            e2e_ms = median_ms(ev)
            del stage, pin

    t_step, t_draft, t_verify = step_ms / 1e3, draft_ms / 1e3, verify_ms / 1e3
    t_e2e = e2e_ms / 1e3 if host_logit_bytes <= HOST_E2E_LIMIT else 0.0
    (t_step, t_e2e, t_draft, t_verify), accepted_all = combine_ranks([t_step, t_e2e, t_draft, t_verify], accepted,
                                                                       world, dev)
    if rank == 0:
        hbm, bf16, src = peaks()
        draft_b = draft_bytes(wl)
        verify_b = verify_bytes(wl, L_h, labels)
        flops = 2 * B * r * V * G
        rounds = world / t_step
        tokens_per_round = accepted_all / (args.steps * world)          # per rank's batch
        tau = tokens_per_round / B                                       # tokens emitted per request
        line = {
            "metric": METRIC, "value": rounds, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": t_step * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": f"synthetic (seeded log-Zipf + Gaussian logits, "
                                                         f"{wl.w_dtype} weights)",
            "config": config_of(wl, world, labels, args.layout, args.ragged),
            "verified_tokens_per_s": accepted_all / (args.steps * t_step),
            "tokens_per_request_per_round": tau,
            "latency_per_token_us": (t_draft + t_verify) / tau * 1e6,
            "draft_ms": t_draft * 1e3, "verify_ms": t_verify * 1e3,
            "hbm_gbs_round": (draft_b + verify_b) / t_step / 1e9,
            "roofline": {"kernel": "markov_draft (draft_main_tc: all positions in one cooperative launch; "
                                   "CUDA events around the call)" if tc else
                                   "markov_draft (draft_main_fma + draft_combine per position; CUDA events "
                                   "around the call)",
                         "bound": "hbm", "achieved": draft_b / t_draft / 1e9, "peak": hbm, "unit": "GB/s",
                         "frac": draft_b / t_draft / 1e9 / hbm,
                         "traffic": measured_traffic("draft_main_tc", B * G) if tc else None,
                         "peak_source": src, "algorithmic_bytes": draft_b, "bias_tflops": flops / t_draft / 1e12,
                         "frac_of_nominal_8TBs": draft_b / t_draft / 8e12},
            "roofline_verify": {"kernel": "verify (verify_stream + verify_stream_finalize, timed together)",
                                "bound": "hbm", "achieved": verify_b / t_verify / 1e9, "peak": hbm, "unit": "GB/s",
                                "frac": verify_b / t_verify / 1e9 / hbm,
                                "traffic": measured_traffic("verify_stream", verify_b),
                                "algorithmic_bytes": verify_b},
            "warm_l2": {"ms_per_step": warm_step_ms, "draft_ms": warm_draft_ms, "rounds_per_s": 1e3 / warm_step_ms},
            "back_to_back": b2b,
            "graph_t2": None if graph_ms is None else {"ms_per_round": graph_ms, "rounds_per_s": 1e3 / graph_ms,
                         "round": "markov_draft -> prefix_schedule_t2 (capacity from step t-2, device ring) -> "
                                  "verify, captured once as a CUDA graph and replayed; L2 flushed between replays"},
            "e2e": ({"value": world / t_e2e, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
                    if host_logit_bytes <= HOST_E2E_LIMIT else
                    {"value": None, "unit": UNIT, "h2d_bytes_per_step": None, "d2h_bytes_per_step": None,
                     "note": f"inputs of {host_logit_bytes / 1e9:.1f} GB per step are not staged in pinned memory"}),
            "gpu_launches": n_launch * args.steps,
            "clocks": clocks,
            "wall_s_timed_region": tw1 - tw0,
        }
        if not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(wl, labels)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
