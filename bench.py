"""Benchmark of one DSpark draft/verify round on B200 (one JSON line on rank 0).

Workload (BASELINE metric): high concurrency, B=64 requests, gamma=16, V=151936, r=256,
T=0.8, bf16 Markov-head weights, fp32 logits (synthetic, seeded; see inputs.py).

One step = one pass of the whole hot path over one batch:
  markov_draft (16 x [tensor-core main pass + combine])
  -> prefix_schedule (prefix survival + greedy scheduler; flat steps/s table, so the whole
     gamma-block is selected and the verified work is the gamma=16 block)
  -> verify (acceptance, residual/bonus sample, fused TV labels).
Inputs live in HBM when the timed region starts; L2 (126 MB) is flushed by writing a
256 MB buffer before every timed step, outside the timed events.

value       = rounds/s over all ranks (each rank runs its own batch: weak scaling)
e2e         = the same rounds/s through the public API with pinned host buffers: the
              per-step inputs are copied host->device and the step's result (n_acc, y)
              device->host inside the timed region
roofline    = the draft stage (all of its launches) against measured HBM copy bandwidth,
              algorithmic bytes B*gamma*V*4 (read U) + gamma*r*V*2 (W2 per step) +
              B*gamma*V*4 (write l_d); the verify kernel is reported beside it
              (B*gamma*V*4 + B*(gamma+1)*V*4 bytes)
cpu_baseline= the CPU oracle on a bounded sample of requests of the same workload

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
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


def workload_bytes(wl):
    B, G, V, r = wl.B, wl.gamma, wl.V, wl.r
    draft = B * G * V * 4 + G * r * V * 2 + B * G * V * 4
    verify = B * G * V * 4 + B * (G + 1) * V * 4
    flops = 2 * B * r * V * G
    return draft, verify, flops


def config_of(wl, n):
    return {"workload": f"{wl.name}: B={wl.B} requests, gamma={wl.gamma}, V={wl.V}, r={wl.r}, T={wl.T}, "
                        f"bf16 W1/W2, fp32 log-Zipf+Gaussian logits",
            "B_per_gpu": wl.B, "gamma": wl.gamma, "V": wl.V, "r": wl.r, "T": wl.T,
            "parallelism": f"replicas over {n} GPU(s), no data-path collective",
            "l2_policy": "256 MB write before every timed step (outside the timed events)",
            "step": "markov_draft -> prefix_schedule (flat sps, full block) -> verify (+TV labels)"}


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


def cpu_baseline(wl, n_req, d=None):
    """The oracle on n_req requests of the workload: one full round, scaled to the whole batch."""
    import oracle as O
    from speculative_decoding_04_b200 import inputs

    threads = os.cpu_count() or 1
    reqs = list(range(n_req))
    U, lt = inputs.logits(wl, reqs)
    W1, W2 = inputs.weights(wl)
    x0 = inputs.tokens(wl)[reqs]
    u_draft, u_acc, u_res = (a[reqs] for a in inputs.uniforms(wl))
    c = inputs.confidences(wl)
    t0 = time.perf_counter()
    x, ld, _ = O.markov_draft(U, W1, W2, x0, u_draft, wl.T)
    sch = O.prefix_schedule(c, np.ones(wl.D_max + 1), wl.D_max)
    O.verify(ld, lt, x, sch["L"][reqs], u_acc, u_res, wl.T)
    O.tv_labels(ld, lt[:, :wl.gamma], wl.T)
    dt = time.perf_counter() - t0
    per_round = dt * wl.B / n_req
    return {"value": 1.0 / per_round, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{n_req} of {wl.B} requests, one full round (draft, schedule, verify, labels), "
                      f"{dt:.1f} s, scaled by {wl.B}/{n_req} (requests are independent)"}


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


def run_reference(args, wl, rank, world):
    # the CPU oracle is the reference arm; rank 0 alone runs it
    if rank != 0:
        return
    steps = []
    n_req = 2
    for i in range(args.warmup + args.steps):
        cb = cpu_baseline(wl, n_req)
        if i >= args.warmup:
            steps.append(1.0 / cb["value"])
    t = statistics.mean(steps)
    line = {"impl": "reference", "metric": METRIC, "value": 1.0 / t, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded, see inputs.py)",
            "config": config_of(wl, args.gpus),
            "cpu_baseline": {"value": 1.0 / t, "unit": UNIT, "cores": cb["cores"], "kind": "oracle",
                             "sample": cb["sample"]},
            "e2e": {"value": 1.0 / t, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="dspark", choices=["dspark", "reference"])
    ap.add_argument("--workload", default="high_concurrency", choices=["high_concurrency", "profile"],
                    help="profile: B=64, gamma=4 (same kernels as the headline, ~0.6 GB on the device) for ncu captures")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the CPU oracle timing (after the GPU timing)")
    ap.add_argument("--cpu-requests", type=int, default=4)
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")

    from speculative_decoding_04_b200 import inputs

    wl = inputs.HIGH_CONCURRENCY
    if args.workload == "profile":
        wl = wl.with_(name="profile", B=64, gamma=4)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if args.impl == "reference":
        return run_reference(args, wl, rank, world)

    import torch
    import torch.distributed as dist

    from speculative_decoding_04_b200 import build
    build.build()
    from speculative_decoding_04_b200 import dspark as D

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    # ---------------------------------------------------------------- inputs (each rank its own batch)
    d = inputs.full_inputs(rank_workload(wl, rank))
    d["U"] = d["U"].transpose(1, 0, 2)      # the draft's base logits are position-major [gamma, B, V]
    pin = {k: torch.from_numpy(np.ascontiguousarray(v)).pin_memory()
           for k, v in d.items() if k in ("U", "lt", "x0", "u_draft", "u_acc", "u_res", "c")}
    W1 = torch.from_numpy(d["W1"]).to(torch.bfloat16).to(dev)
    W2 = torch.from_numpy(d["W2"]).to(torch.bfloat16).to(dev)
    dv = {k: v.to(dev) for k, v in pin.items()}
    B, G, V, r = wl.B, wl.gamma, wl.V, wl.r
    sps = torch.ones(B * G + 1, dtype=torch.float64, device=dev)       # flat: every drafted token is worth verifying
    x = torch.empty((B, G), dtype=torch.int32, device=dev)
    ld = torch.empty((G, B, V), dtype=torch.float32, device=dev)
    fl = torch.zeros(B, dtype=torch.int32, device=dev)
    L = torch.empty(B, dtype=torch.int32, device=dev)
    theta = torch.empty(1, dtype=torch.float64, device=dev)
    n_acc = torch.empty(B, dtype=torch.int32, device=dev)
    y = torch.empty((B, G + 1), dtype=torch.int32, device=dev)
    c_star = torch.empty((B, G), dtype=torch.float32, device=dev)
    ws_d = D.workspace(D.WS_DRAFT, B, G, V, r, dev)
    ws_v = D.workspace(D.WS_VERIFY, B, G, V, 0, dev)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(device=dev)
    D.set_option("draft_fused", 1)  # the draft's gamma positions in one cooperative launch
    n_launch = 1 + 1 + 2  # draft; schedule; verify: stream + finalize

    def round_(src):
        D.markov_draft(src["U"], W1, W2, src["x0"], src["u_draft"], wl.T, x_out=x, ld_out=ld, flags=fl, ws=ws_d,
                       stream=stream)
        D.prefix_schedule(src["c"], sps, B * G, D.SCHED_ARGMAX, L_out=L, theta_out=theta, flags=fl, want_a=False,
                          stream=stream)
        D.verify(ld, src["lt"], x, L, src["u_acc"], src["u_res"], wl.T, n_acc=n_acc, y_out=y, c_star=c_star,
                 flags=fl, ws=ws_v, stream=stream)

    def barrier():
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    clk = Clocks(local)      # sampling starts before the warm-up so that it covers the timed region
    time.sleep(0.5)
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            flush.fill_(1.0)
            round_(dv)
        barrier()
        tw0 = time.perf_counter()
        accepted = 0
        acc_dev = torch.zeros((), dtype=torch.int64, device=dev)
        for i in range(args.steps):
            flush.fill_(float(i))
            ev[i][0].record(stream)
            D.markov_draft(dv["U"], W1, W2, dv["x0"], dv["u_draft"], wl.T, x_out=x, ld_out=ld, flags=fl, ws=ws_d,
                           stream=stream)
            ev[i][1].record(stream)
            D.prefix_schedule(dv["c"], sps, B * G, D.SCHED_ARGMAX, L_out=L, theta_out=theta, flags=fl, want_a=False,
                              stream=stream)
            D.verify(ld, dv["lt"], x, L, dv["u_acc"], dv["u_res"], wl.T, n_acc=n_acc, y_out=y, c_star=c_star,
                     flags=fl, ws=ws_v, stream=stream)
            ev[i][2].record(stream)
            acc_dev += n_acc.sum() + B
        barrier()
        tw1 = time.perf_counter()
        clocks = clk.stop()
        accepted = int(acc_dev.item())
        step_ms = [ev[i][0].elapsed_time(ev[i][2]) for i in range(args.steps)]
        draft_ms = [ev[i][0].elapsed_time(ev[i][1]) for i in range(args.steps)]

        # verify alone, timed live around its one launch (same inputs, after a flush)
        vt = []
        for i in range(args.steps):
            flush.fill_(float(i))
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            D.verify(ld, dv["lt"], x, L, dv["u_acc"], dv["u_res"], wl.T, n_acc=n_acc, y_out=y, c_star=c_star,
                     flags=fl, ws=ws_v, stream=stream)
            e1.record(stream)
            vt.append((e0, e1))
        barrier()
        verify_ms = [a.elapsed_time(b) for a, b in vt]

        # end to end through the public API with pinned host buffers
        n_out = torch.empty_like(n_acc, device="cpu").pin_memory()
        y_out = torch.empty_like(y, device="cpu").pin_memory()
        e2e = []
        h2d = sum(v.numel() * v.element_size() for v in pin.values())
        d2h = n_out.numel() * 4 + y_out.numel() * 4
        stage = {k: torch.empty_like(v) for k, v in dv.items()}
        for i in range(args.warmup + args.steps):
            flush.fill_(float(i))
            barrier()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for k in stage:
                stage[k].copy_(pin[k], non_blocking=True)
            round_(stage)
            n_out.copy_(n_acc, non_blocking=True)
            y_out.copy_(y, non_blocking=True)
            e1.record(stream)
            e1.synchronize()
            if i >= args.warmup:
                e2e.append(e0.elapsed_time(e1))

    t_step = statistics.mean(step_ms) / 1e3
    t_e2e = statistics.mean(e2e) / 1e3
    t_draft = statistics.mean(draft_ms) / 1e3
    t_verify = statistics.mean(verify_ms) / 1e3
    (t_step, t_e2e, t_draft, t_verify), accepted_all = combine_ranks([t_step, t_e2e, t_draft, t_verify], accepted,
                                                                       world, dev)

    if rank == 0:
        hbm, bf16, src = peaks()
        draft_b, verify_b, flops = workload_bytes(wl)
        rounds = world / t_step
        line = {
            "metric": METRIC, "value": rounds, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": t_step * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded log-Zipf + Gaussian logits, bf16 weights)",
            "config": config_of(wl, world),
            "verified_tokens_per_s": accepted_all / (args.steps * t_step),
            "draft_ms": t_draft * 1e3, "verify_ms": t_verify * 1e3,
            "hbm_gbs_round": (draft_b + verify_b) / t_step / 1e9,
            "roofline": {"kernel": f"markov_draft (draft_main_tc<64>: {G} positions in one cooperative launch, "
                                   "timed with CUDA events around the call)",
                         "bound": "hbm", "achieved": draft_b / t_draft / 1e9, "peak": hbm, "unit": "GB/s",
                         "frac": draft_b / t_draft / 1e9 / hbm,
                         "traffic": measured_traffic("draft_main_tc", B * G),
                         "peak_source": src, "algorithmic_bytes": draft_b, "bias_tflops": flops / t_draft / 1e12,
                         "frac_of_nominal_8TBs": draft_b / t_draft / 8e12},
            "roofline_verify": {"kernel": "verify (verify_stream + verify_stream_finalize, timed together)",
                                "bound": "hbm", "achieved": verify_b / t_verify / 1e9, "peak": hbm, "unit": "GB/s",
                                "frac": verify_b / t_verify / 1e9 / hbm,
                                "traffic": measured_traffic("verify_stream", verify_b),
                                "algorithmic_bytes": verify_b},
            "e2e": {"value": world / t_e2e, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": n_launch * args.steps,
            "clocks": clocks,
            "wall_s_timed_region": tw1 - tw0,
        }
        if not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(wl, args.cpu_requests)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
