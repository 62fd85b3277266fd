"""Chunk-KDA forward benchmark (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload I] [--impl ours|reference]

A step is one chunk-KDA forward over the whole workload (default: the dense
4 x 8192 batch, H = 32, K = V = 128, bf16 q/k/v, fp32 g and beta), inputs
already resident in HBM.  Under torchrun every rank runs its own replica of
the workload (documents and heads are independent; no collective on the data
path), so per-GPU work is fixed and the line reports weak scaling.

`--impl reference` times the fp64 CPU oracle on this host's cores instead
(rank 0 only): the whole workload each step when the run fits a few minutes,
else a bounded sample of it.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "chunk-KDA fwd Mtokens/s at H=32,K=V=128 bf16; TFLOP/s and % of roofline"
UNIT = "Mtokens/s"
BYTES_PER_TOKEN_HEAD = 1540          # q,k,v bf16 768 + g fp32 512 + beta 4 + o bf16 256
FLOPS_PER_TOKEN_HEAD = 180224        # 6 d^2 + 10 C d, d = 128, C = 64 (dense chunk tiles)
FLOPS_PER_TOKEN_HEAD_TRI = 139264    # same, skipping the zero triangles
# the recompute backward: reads q, k, v (768 B), g (512), beta (4) and dO (256 B); writes dq, dk, dv
# (768 B), dg (512) and dbeta (4) -- 2824 B per (token, head), each tensor once
BWD_BYTES_PER_TOKEN_HEAD = 2824
FALLBACK_HBM_GBS = 6650.0


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), float(j.get("bf16_tflops", 1590.0)), "measured"
    return FALLBACK_HBM_GBS, 1590.0, "fallback"


FWD_KERNEL_SOURCES = ("kda_fwd_pipe.cu", "kda_tc.cuh", "kda_common.cuh")


def kernel_source_hash() -> str:
    """Hash of the sources of the forward kernel whose DRAM traffic profiles/traffic.json records."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "chunked_gated_delta_12_b200", "csrc")
    for name in FWD_KERNEL_SOURCES:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload_name: str):
    """DRAM bytes per launch from a committed ncu capture, if the kernel sources still match."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        j = json.load(f)
    if j.get("kernel_source_hash") != kernel_source_hash():
        return None
    rec = j.get("per_launch_bytes", {}).get(workload_name)
    return None if rec is None else float(rec)


class ClockSampler:
    """nvidia-smi clock/throttle samples while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, dev_index: int):
        self.dev = dev_index
        self.samples = []
        self._stop = threading.Event()
        self._th = None

    def _run(self):
        while not self._stop.is_set():
            try:
                r = subprocess.run(["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}",
                                    "--format=csv,noheader,nounits"], capture_output=True, text=True,
                                   timeout=5)
                parts = [x.strip() for x in r.stdout.strip().split(",")]
                if len(parts) == 7:
                    self.samples.append(parts)
            except Exception:
                pass
            self._stop.wait(0.05)

    def __enter__(self):
        self._th = threading.Thread(target=self._run, daemon=True)
        self._th.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        self._th.join(timeout=10)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(s[0]) for s in self.samples if s[0].replace(".", "").isdigit()]
        mx = [float(s[1]) for s in self.samples if s[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for s in self.samples for i in range(4) if s[3 + i].lower() == "active"})
        pw = [float(s[2]) for s in self.samples if s[2].replace(".", "").isdigit()]
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(self.samples),
                "power_w": float(np.median(pw)) if pw else None}


def dist_setup(n_gpus: int):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def max_over_ranks(value: float, device=None) -> float:
    """The largest `value` across the ranks of the default process group (the
    value itself when not distributed).  Used for device times, so the slowest
    rank sets the whole-job throughput."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(tokens_per_rank: int, world: int, ms_per_step: float) -> float:
    """Mtokens/s of the whole job: every rank processes its own replica of the workload."""
    return tokens_per_rank * world / (ms_per_step * 1e-3) / 1e6


def oracle_rows(d, tokens: int | None):
    """The oracle's inputs for the first `tokens` tokens of every document (all of them if None),
    as fp32 arrays and the matching cu_seqlens."""
    from chunked_gated_delta_12_b200.inputs import bf16_bits_to_f32
    cu = np.asarray(d["cu_seqlens"], dtype=np.int64)
    if tokens is None:
        idx = np.arange(int(cu[-1]))
        cu_s = cu
    else:
        lens = np.minimum(np.diff(cu), tokens)
        idx = np.concatenate([np.arange(cu[i], cu[i] + lens[i]) for i in range(len(lens))])
        cu_s = np.concatenate([[0], np.cumsum(lens)])
    f = lambda key: bf16_bits_to_f32(d[key][idx]).reshape(d[key][idx].shape)
    return (f("q"), f("k"), f("v"), np.ascontiguousarray(d["g"][idx]), np.ascontiguousarray(d["beta"][idx]),
            cu_s.astype(np.int32))


def oracle_time(inputs, n_threads: int) -> float:
    """Seconds the fp64 oracle, as it stands, takes for one pass over `inputs` (oracle_rows)."""
    import oracle
    q, k, v, g, b, cu = inputs
    t0 = time.perf_counter()
    oracle.kda_fwd(q, k, v, g, b, cu, n_threads=n_threads)
    return time.perf_counter() - t0


def oracle_plan(w, d, cores: int, budget_s: float):
    """Inputs for one oracle step: the whole workload if one pass fits `budget_s` seconds, else the
    first n tokens of every document (all chains kept), n sized from a calibration run."""
    probe = oracle_rows(d, 64)
    per_tok = oracle_time(probe, cores) / int(probe[-1][-1])
    if per_tok * w.T <= budget_s:
        return oracle_rows(d, None), w.T, "the whole workload"
    n = max(64, int(budget_s / per_tok / w.n_docs))
    inputs = oracle_rows(d, n)
    return inputs, int(inputs[-1][-1]), f"the first {n} tokens of each of the {w.n_docs} documents"


def cpu_baseline(w, d, target_s: float = 10.0) -> dict:
    """The fp64 oracle as it stands, on this host's cores: the whole workload (every chain, every
    token) when one pass takes under a minute, else a bounded sample of it, repeated until
    `target_s` seconds of wall time have been spent."""
    cores = os.cpu_count() or 1
    inputs, tokens, what = oracle_plan(w, d, cores, budget_s=60.0)
    total, runs = 0.0, 0
    while total < target_s or runs == 0:
        total += oracle_time(inputs, cores)
        runs += 1
    rate = runs * tokens / total / 1e6
    used = min(cores, w.n_docs * w.H)       # threads over independent (document, head) chains
    return {"value": rate, "unit": UNIT, "cores": used, "kind": "oracle",
            "sample": f"{what} ({tokens} tokens x {w.H} heads, {w.n_docs * w.H} chains), {runs} run(s), "
                      f"{total:.1f} s"}


def run_reference(args, w, d):
    """fp64 oracle on the host cores: each step one pass over the workload (the whole workload when
    every step of the run fits about two and a half minutes, else the same sample each step)."""
    cores = os.cpu_count() or 1
    budget = 150.0 / max(1, args.steps + args.warmup)
    inputs, tokens, what = oracle_plan(w, d, cores, budget_s=budget)
    for _ in range(args.warmup):
        oracle_time(inputs, cores)
    times = [oracle_time(inputs, cores) for _ in range(args.steps)]
    total = sum(times)
    value = args.steps * tokens / total / 1e6
    sample = (f"{what} of {w.name} ({tokens} tokens x {w.H} heads, {w.n_docs * w.H} independent chains, "
              f"fp64 token recurrence)")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": headline_config(w, 1),
            "cpu_baseline": {"kind": "oracle", "value": value, "unit": UNIT,
                             "cores": min(cores, w.n_docs * w.H), "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    if tokens != w.T:
        line["config"]["sample_tokens"] = tokens
    print(json.dumps(line), flush=True)


def headline_config(w, world: int) -> dict:
    gb = w.T * w.H * BYTES_PER_TOKEN_HEAD / 1e9
    l2 = (f"inputs and output {gb:.2f} GB per step > 126 MB L2; no flush" if gb * 1e3 > 126
          else f"inputs and output {gb * 1e3:.1f} MB per step fit the 126 MB L2; not flushed (small case)")
    return dict(w.describe(), l2=l2, parallelism=f"replicas x{world}" if world > 1 else "single GPU")


def bench_backward(kda, steps: int, dev, stream, barrier, shape=None) -> dict:
    """Device time of kda_chunk_bwd on the packed forward+backward workload (16 documents,
    H = 32), or on a dense DOCSxLEN:H `shape`, inputs resident, workspace allocated once; max over
    ranks."""
    import torch
    from chunked_gated_delta_12_b200.inputs import custom_workload, generate, workload
    if shape:
        docs_len, heads = shape.split(":")
        n_docs, doc_len = (int(x) for x in docs_len.split("x"))
        wb = custom_workload(f"dense_{n_docs}x{doc_len}_H{heads}", [doc_len] * n_docs, int(heads), seed=20264)
    else:
        wb = workload(4)
    db = generate(wb, with_grad=True)
    t = {}
    for key in ("q", "k", "v", "do"):
        t[key] = torch.from_numpy(db[key].view(np.int16)).view(torch.bfloat16).to(dev)
    for key in ("g", "beta", "cu_seqlens"):
        t[key] = torch.from_numpy(db[key]).to(dev)
    ws = torch.empty(kda.bwd_workspace_bytes(wb.n_docs, wb.T, wb.H), dtype=torch.uint8, device=dev)

    def run():
        kda.kda_chunk_bwd(t["q"], t["k"], t["v"], t["g"], t["beta"], t["cu_seqlens"], t["do"], workspace=ws,
                          stream=stream)

    run()
    kda.device_status(stream)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(steps):
        run()
    e1.record(stream)
    torch.cuda.synchronize()
    kda.device_status(stream)
    ms = max_over_ranks(e0.elapsed_time(e1) / steps, dev)
    hbm_peak, _, peak_kind = peaks()
    alg = wb.T * wb.H * BWD_BYTES_PER_TOKEN_HEAD
    gbs = alg / (ms * 1e-3) / 1e9
    return {"workload": wb.name, "T": wb.T, "H": wb.H, "ms_per_launch": ms, "launches": steps,
            "Mtokens_per_s": wb.T / (ms * 1e-3) / 1e6, "workspace_bytes": ws.numel(),
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm_peak, "unit": "GB/s", "frac": gbs / hbm_peak,
                         "peak_source": peak_kind, "algorithmic_bytes_per_launch": alg,
                         "bytes_per_token_head": BWD_BYTES_PER_TOKEN_HEAD}}


def bench_workloads(kda, steps: int, dev, stream, barrier) -> dict:
    """Device time of the forward on the other full-size workloads, inputs resident, max over
    ranks: one document of 65536 tokens with H = 32 (32 chains of 1024 chunks) through
    kda_chunk_fwd and through kda_chunk_fwd_long with its default segment count (workspace
    allocated once), and the 16 packed documents (H = 32) through kda_chunk_fwd."""
    import torch
    from chunked_gated_delta_12_b200.inputs import generate, workload
    hbm_peak, _, peak_kind = peaks()
    res = {}
    for idx in (3, 4):
        wl = workload(idx)
        dl = generate(wl, with_grad=False)
        t = {}
        for key in ("q", "k", "v"):
            t[key] = torch.from_numpy(dl[key].view(np.int16)).view(torch.bfloat16).to(dev)
        for key in ("g", "beta", "cu_seqlens"):
            t[key] = torch.from_numpy(dl[key]).to(dev)
        del dl
        out = torch.empty_like(t["q"])
        split = kda.use_split(wl.n_docs, wl.T, wl.H)
        ws_split = torch.empty(max(kda.split_workspace_bytes(wl.n_docs, wl.T, wl.H), 256), dtype=torch.uint8,
                               device=dev) if split else None
        # kda_chunk_fwd as a user calls it (few chains: routed to kda_chunk_fwd_split), and unsplit
        runs = {"kda_chunk_fwd": lambda: kda.kda_chunk_fwd(t["q"], t["k"], t["v"], t["g"], t["beta"],
                                                           t["cu_seqlens"], out=out, stream=stream,
                                                           workspace=ws_split)}
        if split:
            runs["kda_chunk_fwd_unsplit"] = lambda: kda.kda_chunk_fwd(t["q"], t["k"], t["v"], t["g"], t["beta"],
                                                                      t["cu_seqlens"], out=out, stream=stream,
                                                                      split=False)
        entry = {"T": wl.T, "H": wl.H, "n_docs": wl.n_docs, "chains": wl.n_docs * wl.H, "split": split}
        if wl.n_docs == 1:
            P = kda.long_segments(wl.T, wl.H)
            ws = torch.empty(max(kda.long_workspace_bytes(wl.T, wl.H, P), 256), dtype=torch.uint8, device=dev)
            runs["kda_chunk_fwd_long"] = lambda: kda.kda_chunk_fwd_long(t["q"], t["k"], t["v"], t["g"], t["beta"],
                                                                        out=out, segments=P, workspace=ws,
                                                                        stream=stream)
            entry.update(segments=P, workspace_bytes=ws.numel())
        best = None
        for name, run in runs.items():
            for _ in range(3):
                run()
            kda.device_status(stream)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            barrier()
            torch.cuda.synchronize()
            e0.record(stream)
            for _ in range(steps):
                run()
            e1.record(stream)
            torch.cuda.synchronize()
            kda.device_status(stream)
            ms = max_over_ranks(e0.elapsed_time(e1) / steps, dev)
            alg = wl.T * wl.H * BYTES_PER_TOKEN_HEAD
            gbs = alg / (ms * 1e-3) / 1e9
            entry[name] = {"ms_per_call": ms, "Mtokens_per_s": wl.T / (ms * 1e-3) / 1e6, "launches": steps,
                           "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm_peak, "unit": "GB/s",
                                        "frac": gbs / hbm_peak, "peak_source": peak_kind,
                                        "algorithmic_bytes_per_launch": alg}}
            if best is None or ms < entry[best]["ms_per_call"]:
                best = name
        entry["best_public_path"] = best
        res[wl.name] = entry
        del t, out
        torch.cuda.empty_cache()
    return res


DECODE_DOCS = 256                    # one decoding step of 256 sequences x 32 heads, states in place
STATE_BYTES = 2 * 128 * 128 * 4      # fp32 state read and written per chain


def bench_decode(kda, steps: int, dev, stream, barrier) -> dict:
    """Device time of kda_recurrent_fwd for one decoding step (one token for each of 256
    documents, H = 32) with the 128 x 128 fp32 states updated in place; the states (537 MB) are
    larger than L2.  Bound: HBM, STATE_BYTES + BYTES_PER_TOKEN_HEAD per chain."""
    import torch
    from chunked_gated_delta_12_b200.inputs import custom_workload, generate
    wd = custom_workload("decode_256x1_H32", [1] * DECODE_DOCS, 32, seed=20265)
    dd = generate(wd)
    t = {}
    for key in ("q", "k", "v"):
        t[key] = torch.from_numpy(dd[key].view(np.int16)).view(torch.bfloat16).to(dev)
    for key in ("g", "beta", "cu_seqlens"):
        t[key] = torch.from_numpy(dd[key]).to(dev)
    gen = torch.Generator(device=dev).manual_seed(20266)
    state = torch.randn(wd.n_docs, wd.H, 128, 128, device=dev, generator=gen) * 0.1
    out = torch.empty_like(t["q"])

    def run():
        kda.kda_recurrent_fwd(t["q"], t["k"], t["v"], t["g"], t["beta"], t["cu_seqlens"], out=out, stream=stream,
                              initial_state=state, final_state=state)

    for _ in range(3):
        run()
    kda.device_status(stream)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(steps):
        run()
    e1.record(stream)
    torch.cuda.synchronize()
    kda.device_status(stream)
    ms = max_over_ranks(e0.elapsed_time(e1) / steps, dev)
    hbm_peak, _, peak_kind = peaks()
    alg = wd.n_docs * wd.H * (STATE_BYTES + BYTES_PER_TOKEN_HEAD)
    gbs = alg / (ms * 1e-3) / 1e9
    return {"workload": wd.name, "T": wd.T, "H": wd.H, "ms_per_launch": ms, "launches": steps,
            "Mtokens_per_s": wd.T / (ms * 1e-3) / 1e6,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm_peak, "unit": "GB/s", "frac": gbs / hbm_peak,
                         "peak_source": peak_kind, "algorithmic_bytes_per_launch": alg}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", type=int, default=2)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--bwd-steps", type=int, default=3,
                    help="timed launches of the recompute backward on the packed forward+backward "
                         "workload, reported under 'backward' (0 skips it)")
    ap.add_argument("--dec-steps", type=int, default=20,
                    help="timed launches of the token-by-token kernel on one decoding step of 256 "
                         "sequences, reported under 'decode' (0 skips it)")
    ap.add_argument("--fwd-steps", type=int, default=10,
                    help="timed forward calls on each of the other full-size workloads (one document of "
                         "65536 tokens, also split by kda_chunk_fwd_long; 16 packed documents), reported "
                         "under 'workloads' (0 skips them)")
    ap.add_argument("--bwd-shape", default=None,
                    help="DOCSxLEN:H -- run the backward on a custom dense workload instead (profiling)")
    ap.add_argument("--shape", default=None,
                    help="DOCSxLEN:H -- a custom dense workload with the same distributions "
                         "(e.g. 4x2048:32 for a profiling case larger than L2)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    from chunked_gated_delta_12_b200.inputs import custom_workload, generate, workload
    if args.shape:
        docs_len, heads = args.shape.split(":")
        n_docs, doc_len = (int(x) for x in docs_len.split("x"))
        w = custom_workload(f"dense_{n_docs}x{doc_len}_H{heads}", [doc_len] * n_docs, int(heads), seed=20262)
    else:
        w = workload(args.workload)

    if args.impl == "reference":
        if int(os.environ.get("RANK", "0")) != 0:
            return
        d = generate(w)
        run_reference(args, w, d)
        return

    import torch
    import chunked_gated_delta_12_b200 as kda
    world, rank, local = dist_setup(args.gpus)
    dev = torch.device("cuda", torch.cuda.current_device())
    d = generate(w)
    host = {}
    for key in ("q", "k", "v"):
        host[key] = torch.from_numpy(d[key].view(np.int16)).view(torch.bfloat16).pin_memory()
    host["g"] = torch.from_numpy(d["g"]).pin_memory()
    host["beta"] = torch.from_numpy(d["beta"]).pin_memory()
    host["cu_seqlens"] = torch.from_numpy(d["cu_seqlens"]).pin_memory()
    dv = {key: t.to(dev) for key, t in host.items()}
    out = torch.empty_like(dv["q"])
    stream = torch.cuda.current_stream()

    def step():
        kda.kda_chunk_fwd(dv["q"], dv["k"], dv["v"], dv["g"], dv["beta"], dv["cu_seqlens"], out=out,
                          stream=stream)

    for _ in range(args.warmup):
        step()
    kda.device_status(stream)
    torch.cuda.synchronize()

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    # timed region: K steps, events on the launching stream (one kernel launch per step)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    smi_index = int(os.environ.get("CUDA_VISIBLE_DEVICES", str(local)).split(",")[local]) \
        if os.environ.get("CUDA_VISIBLE_DEVICES") else local
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(smi_index) as clk:
        ev[0].record(stream)
        for i in range(args.steps):
            step()
            ev[i + 1].record(stream)
        torch.cuda.synchronize()
    barrier()
    kda.device_status(stream)
    per_launch_ms = [ev[i].elapsed_time(ev[i + 1]) for i in range(args.steps)]
    elapsed_ms = max_over_ranks(ev[0].elapsed_time(ev[-1]), dev)

    # end to end through the C ABI on host buffers: kda_chunk_fwd_host enqueues the copies of the
    # pinned inputs into a device workspace, the forward and the copy of the output back, on the
    # stream.  A call that kda_chunk_fwd routes through the segment split (few chains) keeps that
    # route: its inputs are copied by torch around the same public call.
    host_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = host_out.numel() * host_out.element_size()
    n_docs = int(host["cu_seqlens"].numel()) - 1
    e2e_split = kda.use_split(n_docs, w.T, w.H)
    ws_host = None if (args.no_e2e or e2e_split) else torch.empty(kda.host_workspace_bytes(n_docs, w.T, w.H),
                                                                  dtype=torch.uint8, device=dev)

    def e2e_step():
        if ws_host is not None:
            kda.kda_chunk_fwd_host(host["q"], host["k"], host["v"], host["g"], host["beta"], host["cu_seqlens"],
                                   host_out, ws_host, stream=stream)
        else:
            for key in host:
                dv[key].copy_(host[key], non_blocking=True)
            step()
            host_out.copy_(out, non_blocking=True)

    if not args.no_e2e:
        e2e_step()   # untimed: first use of the workspace
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(0 if args.no_e2e else args.e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / max(1, args.e2e_steps) if not args.no_e2e else float("nan")
    e2e_ms = max_over_ranks(e2e_ms, dev)

    tokens_all = w.T * world
    ms_step = elapsed_ms / args.steps
    value = whole_job_rate(w.T, world, ms_step)
    hbm_peak, tc_peak, peak_kind = peaks()
    launch_ms = float(np.mean(per_launch_ms))
    alg_bytes = w.T * w.H * BYTES_PER_TOKEN_HEAD
    achieved = alg_bytes / (launch_ms * 1e-3) / 1e9
    tflops = w.T * w.H * FLOPS_PER_TOKEN_HEAD / (launch_ms * 1e-3) / 1e12
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": headline_config(w, world),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                     "frac": achieved / hbm_peak, "traffic": recorded_traffic(w.name),
                     "peak_source": peak_kind, "algorithmic_bytes_per_launch": alg_bytes,
                     "launch_ms": launch_ms},
        "tflops": {"dense_tile": tflops, "triangle_exact": tflops * FLOPS_PER_TOKEN_HEAD_TRI / FLOPS_PER_TOKEN_HEAD,
                   "frac_of_bf16_peak": tflops / tc_peak},
        "gpu_launches": args.steps,
        "clocks": clk.summary(),
        "e2e": {"value": tokens_all / (e2e_ms * 1e-3) / 1e6, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": args.e2e_steps,
                "call": "kda_chunk_fwd (torch copies around it, split route)" if e2e_split
                        else "kda_chunk_fwd_host (C ABI on pinned host buffers)"},
    }
    if args.bwd_steps > 0:
        line["backward"] = bench_backward(kda, args.bwd_steps, dev, stream, barrier, args.bwd_shape)
    if args.dec_steps > 0:
        line["decode"] = bench_decode(kda, args.dec_steps, dev, stream, barrier)
    if args.fwd_steps > 0:
        line["workloads"] = bench_workloads(kda, args.fwd_steps, dev, stream, barrier)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, d)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
