#!/usr/bin/env python
"""Benchmark of the hot path: one serving step per GPU.

A step is one pass of every hot-path kernel over one batch of synthetic input,
the two halves of the measured metric together:

* causal prefill, B=4 H=32 N=4096 d=128 bf16, contiguous [B,H,N,d]
  (tcgen05 tensor-core kernel; tensor-bound);
* paged decode, 64 sequences x 32 heads x d=128 bf16, seq_lens U[512, 8192],
  page_size 16, pages shuffled over the pool (split-K kernel + log-sum-exp
  combine; HBM-bound).

``value`` is the fraction of one B200's roofline the step reaches, in percent:
100 * (prefill FLOPs / peak FLOP/s + decode bytes / peak HBM B/s) / step time,
summed over GPUs (each GPU runs an independent replica: weak scaling).  The
per-kernel figures (TFLOP/s, GB/s, each against its measured peak) are in the
same JSON line.  Peaks come from MEASURED_PEAKS.json at the repository root.

Usage:  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
For N > 1 launch one process per GPU with torch.distributed.run.
``--impl reference`` times the fp64 CPU oracle on a bounded sample of the same
workload per step (rank 0 only).
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "paged decode KV GB/s & causal prefill TFLOP/s, % of B200 roofline"
UNIT = "% of B200 roofline (prefill FLOPs at bf16 peak + decode KV bytes at HBM peak; summed over GPUs)"
WORKLOAD = ("serving step: causal prefill B=4 H=32 N=4096 d=128 bf16 + paged decode 64 seqs x "
            "32 heads d=128 bf16, seq_lens U[512,8192], page_size 16")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

PREFILL_SRC = ["prefill_sm100.cu", "sm100_ptx.cuh", "common.cuh"]
DECODE_SRC = ["decode.cu", "common.cuh"]


# ---------------------------------------------------------------------------
# host-side helpers (also exercised by the CPU multi-rank tests)
# ---------------------------------------------------------------------------

def load_peaks(path=os.path.join(ROOT, "MEASURED_PEAKS.json")):
    try:
        with open(path) as f:
            m = json.load(f)
        return {k: float(m[k]) for k in FALLBACK_PEAKS}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def source_hash(names) -> str:
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "paged_kv_cache_exact_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, src_names, units_now: float):
    """DRAM bytes per launch from the committed ncu summary, scaled to this
    launch's units; None if absent or the kernel source changed since."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            t = json.load(f)[kernel]
    except (OSError, KeyError, ValueError):
        return None
    if t.get("source_sha") != source_hash(src_names):
        return None
    return t["dram_bytes_per_launch"] * units_now / t["units_per_launch"]


SUSTAINED_AFTER_S = 1.0


def tensor_peak(peaks, timed_s, peak_src="measured"):
    """The bf16 tensor peak a kernel's TFLOP/s is measured against, and why.

    A kernel timed inside a region of at least SUSTAINED_AFTER_S seconds of
    back-to-back work runs under the 1 kW power cap: the sustained figure
    applies.  A shorter region runs at burst clocks: the burst figure."""
    if timed_s >= SUSTAINED_AFTER_S:
        return peaks["bf16_tflops_sustained"], (
            f"MEASURED_PEAKS.json bf16_tflops_sustained ({peak_src}): timed region "
            f"{timed_s:.3f} s >= {SUSTAINED_AFTER_S:.0f} s of back-to-back work")
    return peaks["bf16_tflops"], (
        f"MEASURED_PEAKS.json bf16_tflops, burst ({peak_src}): timed region {timed_s:.3f} s "
        f"< {SUSTAINED_AFTER_S:.0f} s")


def roofline_value(prefill_flops, decode_bytes, step_s, peaks, n_ranks=1):
    t_roof = prefill_flops / (peaks["bf16_tflops"] * 1e12) + decode_bytes / (peaks["hbm_gbs"] * 1e9)
    return 100.0 * n_ranks * t_roof / step_s


class ClockSampler:
    """nvidia-smi clock/throttle sampling while the timed region runs."""
    QUERY = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def mark(self, begin: bool):
        if begin:
            self.t0 = time.time()
        else:
            self.t1 = time.time()

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        rows = []
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 10:
                continue
            try:
                ts = time.mktime(time.strptime(f[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                rows.append((ts, float(f[2]), float(f[3]), f[6:10]))
            except ValueError:
                continue
        inside = [r for r in rows if self.t0 - 1 <= r[0] <= self.t1 + 1] or rows
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in inside for i, v in enumerate(r[3]) if v == "Active"})
        return {"sm_mhz": statistics.median(r[1] for r in inside),
                "sm_max_mhz": max(r[2] for r in inside), "reasons": reasons,
                "samples": len(inside)}


def reduce_max(values, dist, device=None):
    """Element-wise max over ranks (identity on one rank)."""
    if dist is None:
        return list(values)
    import torch
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def format_line(d: dict) -> str:
    return json.dumps(d, sort_keys=False)


# ---------------------------------------------------------------------------
# the GPU arm
# ---------------------------------------------------------------------------

def build_step(device):
    """Device-resident inputs of both workloads and a step function."""
    import torch

    from paged_kv_cache_exact_b200 import accounting, api
    from paged_kv_cache_exact_b200.workloads import workload

    pre = workload(2)
    dec = workload(3)
    B, H, N, d = pre.Q.shape
    S = dec.num_seqs
    host = {
        "Q": pre.Q.pin_memory(), "K": pre.K.pin_memory(), "V": pre.V.pin_memory(),
        "q": dec.q.pin_memory(), "table": dec.block_table.pin_memory(),
        "lens": dec.seq_lens.pin_memory(),
    }
    dev = {k: v.to(device, non_blocking=True) for k, v in host.items()}
    dev["k_pages"] = dec.k_pages.to(device)
    dev["v_pages"] = dec.v_pages.to(device)
    dev["O"] = torch.empty_like(dev["Q"])
    dev["out"] = torch.empty_like(dev["q"])
    dev["ws"] = api.workspace_for(S, 32, d, dec.max_seq_len, dec.page_size, device)
    host["O"] = torch.empty(dev["O"].shape, dtype=dev["O"].dtype).pin_memory()
    host["out"] = torch.empty(dev["out"].shape, dtype=dev["out"].dtype).pin_memory()
    torch.cuda.synchronize(device)

    flops = accounting.prefill_flops(B, H, N, N, d, True)
    dbytes = accounting.decode_bytes(dec.seq_lens.tolist(), 32, 32, d,
                                     max_pages=dec.block_table.shape[1])
    max_len = dec.max_seq_len

    def prefill(stream, d=dev):
        api.prefill(d["Q"], d["K"], d["V"], True, pre.scale, out=d["O"], stream=stream)

    def decode(stream, d=dev):
        api.paged(d["q"], dev["k_pages"], dev["v_pages"], d["table"], d["lens"], 16, True,
                  dec.scale, max_seq_len=max_len, out=d["out"], workspace=dev["ws"],
                  stream=stream)

    meta = {"inputs": (pre, dec), "prefill_flops": flops, "decode_bytes": dbytes, "sum_L": int(dec.seq_lens.sum()),
            "decode_units": int(dec.seq_lens.sum()) * 32,
            "h2d": sum(host[k].numel() * host[k].element_size()
                       for k in ("Q", "K", "V", "q", "table", "lens")),
            "d2h": sum(host[k].numel() * host[k].element_size() for k in ("O", "out")),
            "launches_per_step": 1 + (2 if dev["ws"] is not None else 1),
            "pool_bytes": dev["k_pages"].numel() * 2 * 2}
    return prefill, decode, dev, host, meta


def run_gpu(args, rank, world, dist):
    import torch

    local = int(os.environ.get("LOCAL_RANK", "0"))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    from paged_kv_cache_exact_b200 import binding as B

    peaks, peak_src = load_peaks()
    prefill, decode, dev, host, meta = build_step(device)
    stream = torch.cuda.current_stream(device)

    def barrier():
        if dist is not None:
            dist.barrier()

    def step(evs=None):
        if evs is not None:
            evs[0].record(stream)
        prefill(stream)
        if evs is not None:
            evs[1].record(stream)
        decode(stream)
        if evs is not None:
            evs[2].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    st, bits = B.pkv_last_device_error(stream)
    if st != 0:
        raise RuntimeError(f"device error after warm-up: {bits:#x}")

    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.5)
    per = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(device)
    sampler.mark(True)
    t_start.record(stream)
    for k in range(args.steps):
        step(per[k])
    t_end.record(stream)
    torch.cuda.synchronize(device)
    sampler.mark(False)
    barrier()
    clocks = sampler.stop()
    total_ms = t_start.elapsed_time(t_end)
    pre_ms = sum(e[0].elapsed_time(e[1]) for e in per) / args.steps
    dec_ms = sum(e[1].elapsed_time(e[2]) for e in per) / args.steps
    st, bits = B.pkv_last_device_error(stream)
    if st != 0:
        raise RuntimeError(f"device error in the timed region: {bits:#x}")

    # End to end, every step: the step's inputs from pinned host memory, its
    # results back to pinned host memory.  Steps are pipelined over two device
    # buffer sets and three streams: the copy of step i+1's inputs and of step
    # i-1's results overlap step i's kernels (a serving loop would do the same).
    n_e2e = max(3, min(args.steps, 20))
    in_keys, out_keys = ("Q", "K", "V", "q", "table", "lens"), ("O", "out")
    bufs = [dev, {k: torch.empty_like(dev[k]) for k in in_keys + out_keys}]
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev = {(name, b): torch.cuda.Event() for name in ("in", "comp", "out") for b in (0, 1)}
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(device)
    e0.record(stream)
    s_in.wait_event(e0)
    s_out.wait_event(e0)
    for i in range(n_e2e):
        b = i % 2
        d = bufs[b]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev[("comp", b)])        # step i-2 done reading these inputs
            for k in in_keys:
                d[k].copy_(host[k], non_blocking=True)
            ev[("in", b)].record(s_in)
        stream.wait_event(ev[("in", b)])
        if i >= 2:
            stream.wait_event(ev[("out", b)])           # step i-2's results copied out
        prefill(stream, d)
        decode(stream, d)
        ev[("comp", b)].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev[("comp", b)])
            for k in out_keys:
                host[k].copy_(d[k], non_blocking=True)
            ev[("out", b)].record(s_out)
    stream.wait_event(ev[("out", (n_e2e - 1) % 2)])
    stream.wait_event(ev[("in", (n_e2e - 1) % 2)])
    e1.record(stream)
    torch.cuda.synchronize(device)
    barrier()
    e2e_ms = e0.elapsed_time(e1) / n_e2e
    del bufs[1]

    append = measure_append(device, stream, peaks)
    paged_study = measure_paged_study(dev, stream, peaks)
    fp8 = measure_fp8(dev, stream, peaks)
    legs = measure_workload_legs(device, stream, peaks,
                                 cpu=(rank == 0 and world == 1 and not args.no_cpu_baseline))
    total_ms, e2e_ms, pre_ms, dec_ms = reduce_max([total_ms, e2e_ms, pre_ms, dec_ms], dist,
                                                  device)
    ms_step = total_ms / args.steps
    value = roofline_value(meta["prefill_flops"], meta["decode_bytes"], ms_step / 1e3, peaks, world)
    e2e_value = roofline_value(meta["prefill_flops"], meta["decode_bytes"], e2e_ms / 1e3, peaks,
                               world)
    pre_tf = meta["prefill_flops"] / (pre_ms / 1e3) / 1e12
    dec_gbs = meta["decode_bytes"] / (dec_ms / 1e3) / 1e9
    # A tensor-bound kernel is measured against the burst peak unless the timed
    # region lasted long enough for the power cap to set the clocks.
    tpeak, tsrc = tensor_peak(peaks, total_ms / 1e3, peak_src)
    if pre_ms >= dec_ms:
        roof = {"kernel": "prefill_kernel", "bound": "tensor", "achieved": pre_tf,
                "peak": tpeak, "unit": "TFLOP/s", "frac": pre_tf / tpeak,
                "frac_of_burst_peak": pre_tf / peaks["bf16_tflops"],
                "traffic": ncu_traffic("prefill_kernel", PREFILL_SRC, 1.0),
                "peak_source": tsrc}
    else:
        roof = {"kernel": "decode_split_kernel (+ combine)", "bound": "hbm", "achieved": dec_gbs,
                "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": dec_gbs / peaks["hbm_gbs"],
                "traffic": ncu_traffic("decode_split_kernel", DECODE_SRC, meta["decode_units"]),
                "peak_source": f"MEASURED_PEAKS.json hbm_gbs ({peak_src})"}

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16; shuffled page pool with NaN-poisoned decoys)",
        "config": {"workload": WORKLOAD, "parallelism": f"replicas x{world} (no collective)",
                   "prefill": "B=4 H=32 N=4096 d=128 causal, scale 1/sqrt(128)",
                   "decode": f"64 seqs, sum(seq_lens)={meta['sum_L']}, page_size 16, "
                             f"pool {meta['pool_bytes'] / 1e9:.2f} GB",
                   "l2": "inputs larger than L2 (403 MB prefill Q/K/V, "
                         f"{meta['pool_bytes'] / 1e9:.1f} GB KV pool per step)"},
        "prefill": {"ms": pre_ms, "tflops": pre_tf, "frac": pre_tf / peaks["bf16_tflops"],
                    "frac_sustained": pre_tf / peaks["bf16_tflops_sustained"],
                    "frac_of_peak_used": pre_tf / tpeak, "peak_source": tsrc},
        "decode": {"ms": dec_ms, "kv_gbs": dec_gbs, "frac": dec_gbs / peaks["hbm_gbs"]},
        "roofline": roof,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": meta["h2d"],
                "d2h_bytes_per_step": meta["d2h"], "ms_per_step": e2e_ms,
                "note": "pinned host Q/K/V, q, block_table, seq_lens in and O, out back every "
                        "step, pipelined over 2 buffer sets and 3 streams; the KV page pool is "
                        "resident device state"},
        "append": append,
        "workloads": legs,
        "paged_vs_contiguous": paged_study,
        "fp8_qk_prefill": fp8,
        "gpu_launches": args.steps * meta["launches_per_step"],
        "clocks": clocks,
    }
    return line, meta["inputs"]


def append_setup(device, seqs=64, tokens=512, page_size=16, H_kv=32, d=128):
    """A prefill-sized KV append (every sequence writes `tokens` new rows into
    shuffled pages of its own pool); inputs and pool exceed L2."""
    import torch

    gen = torch.Generator().manual_seed(1099)
    rows = seqs * tokens
    pages_per = tokens // page_size
    num_pages = seqs * pages_per
    k_new = torch.randn(rows, H_kv, d, generator=gen).to(torch.bfloat16).to(device)
    v_new = torch.randn(rows, H_kv, d, generator=gen).to(torch.bfloat16).to(device)
    perm = torch.randperm(num_pages, generator=gen).to(torch.int32)
    table = perm.view(seqs, pages_per).contiguous().to(device)
    cu = (torch.arange(seqs + 1, dtype=torch.int32) * tokens).to(device)
    start = torch.zeros(seqs, dtype=torch.int32, device=device)
    k_pages = torch.empty(num_pages, page_size, H_kv, d, dtype=torch.bfloat16, device=device)
    v_pages = torch.empty_like(k_pages)
    from paged_kv_cache_exact_b200 import binding as B

    def run(stream):
        B.paged_kv_append(k_new, v_new, cu, start, table, pages_per, seqs, rows, k_pages, v_pages,
                          num_pages, page_size, H_kv, d, B.PKV_BF16, stream)
    moved = 2 * 2 * rows * H_kv * d * 2           # read K,V rows + write them
    return run, moved, f"{seqs} seqs x {tokens} new tokens, H_kv={H_kv} d={d} bf16, page 16"


def _to_pages(K, page_size, gen):
    """[B, H, N, d] -> ([B*N/ps (+slack) pages, ps, H, d], table [B, N/ps]) over shuffled pages."""
    import torch
    Bn, H, N, d = K.shape
    per = N // page_size
    num_pages = Bn * per
    perm = torch.randperm(num_pages, generator=gen).to(torch.int32)
    table = perm.view(Bn, per)
    pages = torch.empty(num_pages, page_size, H, d, dtype=K.dtype, device=K.device)
    src = K.permute(0, 2, 1, 3).reshape(Bn * per, page_size, H, d)    # logical pages in order
    pages[perm.to(K.device).long()] = src
    return pages, table.to(K.device)


def measure_paged_study(dev, stream, peaks, iters=20):
    """The step's prefill with K/V read through shuffled page tables (16 and
    256 tokens per page) against the contiguous kernel, and the last 512-query
    chunk of each prompt (chunked prefill, bottom-right causal mask)."""
    import torch

    from paged_kv_cache_exact_b200 import accounting, api
    Q, K, V = dev["Q"], dev["K"], dev["V"]
    Bn, H, N, d = Q.shape
    scale = d ** -0.5
    gen = torch.Generator().manual_seed(1098)
    lens = torch.full((Bn,), N, dtype=torch.int32, device=Q.device)

    def timed(fn):
        for _ in range(3):
            fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(iters):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / iters

    O = torch.empty_like(Q)
    flops = accounting.prefill_flops(Bn, H, N, N, d, True)
    out = {"workload": f"prefill B={Bn} H={H} N={N} d={d} causal"}
    out["contiguous_ms"] = timed(lambda: api.prefill(Q, K, V, True, scale, out=O, stream=stream))
    for ps in (256, 16):
        kp, tb = _to_pages(K, ps, gen)
        vp = torch.empty_like(kp)                  # V follows K's table
        per = N // ps
        vsrc = V.permute(0, 2, 1, 3).reshape(Bn * per, ps, H, d)
        vp[tb.reshape(-1).long()] = vsrc
        ms = timed(lambda: api.paged(Q, kp, vp, tb, lens, ps, True, scale, max_seq_len=N,
                                     out=O, stream=stream))
        out[f"paged_ps{ps}_ms"] = ms
        out[f"paged_ps{ps}_vs_contiguous"] = out["contiguous_ms"] / ms
        if ps == 256:
            qc = Q[:, :, N - 512:].contiguous()
            oc = torch.empty_like(qc)
            cms = timed(lambda: api.paged(qc, kp, vp, tb, lens, ps, True, scale, max_seq_len=N,
                                          out=oc, stream=stream))
            cfl = accounting.prefill_flops(Bn, H, 512, N, d, True)
            out["chunked_prefill"] = {"workload": f"last 512 queries of each of {Bn} prompts of "
                                                  f"{N} tokens, H={H}, page 256",
                                      "ms": cms, "tflops": cfl / (cms / 1e3) / 1e12,
                                      "frac": cfl / (cms / 1e3) / 1e12 / peaks["bf16_tflops"]}
        del kp, vp
    out["contiguous_tflops"] = flops / (out["contiguous_ms"] / 1e3) / 1e12
    return out


def measure_fp8(dev, stream, peaks, iters=20):
    """The step's prefill with e4m3 Q and K (per-tensor scales; S = QK^T on the
    FP8 tensor-core path, PV in bf16)."""
    import torch

    from paged_kv_cache_exact_b200 import accounting
    from paged_kv_cache_exact_b200 import binding as B
    Q, K, V = dev["Q"], dev["K"], dev["V"]
    Bn, H, N, d = Q.shape
    qd = float(Q.float().abs().max()) / 448.0
    kd = float(K.float().abs().max()) / 448.0
    Q8 = (Q.float() / qd).to(torch.float8_e4m3fn).view(torch.uint8)
    K8 = (K.float() / kd).to(torch.float8_e4m3fn).view(torch.uint8)
    O = torch.empty_like(V)

    def run():
        B.attn_prefill_fp8qk(Q8, K8, V, O, Bn, H, N, d, True, d ** -0.5, qd, kd, stream)
    for _ in range(3):
        run()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(iters):
        run()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / iters
    tf = accounting.prefill_flops(Bn, H, N, N, d, True) / (ms / 1e3) / 1e12
    return {"workload": f"causal prefill B={Bn} H={H} N={N} d={d}, e4m3 Q/K, bf16 V/O",
            "ms": ms, "tflops": tf, "frac_of_bf16_peak": tf / peaks["bf16_tflops"]}


def _timed_leg(fn, stream, device, min_s=0.4, warmup=3):
    """Time fn() with CUDA events on `stream` over at least `min_s` seconds of
    back-to-back calls (after `warmup` untimed ones), sampling the SM clocks
    over that same region.  Returns (ms per call, calls, clocks)."""
    import torch

    for _ in range(warmup):
        fn()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(device)
    e0.record(stream)
    fn()
    e1.record(stream)
    torch.cuda.synchronize(device)
    iters = max(10, int(min_s * 1e3 / max(e0.elapsed_time(e1), 1e-3)))
    sampler = ClockSampler(device.index or 0)
    sampler.start()
    time.sleep(0.3)
    torch.cuda.synchronize(device)
    sampler.mark(True)
    e0.record(stream)
    for _ in range(iters):
        fn()
    e1.record(stream)
    torch.cuda.synchronize(device)
    sampler.mark(False)
    clocks = sampler.stop()
    return e0.elapsed_time(e1) / iters, iters, clocks


def gqa_decode_workload():
    """Grouped-query decode: 64 sequences x 64 query heads over 8 kv heads,
    d=128 bf16, seq_lens U[512, 8192], 16-token pages (the pages' Llama-3.1-70B
    head grouping, "Attention Variants: MHA, GQA, MQA", on the paged-decode
    length mix)."""
    from paged_kv_cache_exact_b200.workloads import make_paged
    return make_paged(2003, (512, 8192, 64), 64, 128, 16, q_len=1, H_kv=8, decoys=64)


def measure_workload_legs(device, stream, peaks, cpu=True):
    """The other workloads, each timed alone: paged decode with 256-token
    pages (16 seqs, seq_lens U[600, 32768], seq 0 = 600 tokens on pages
    [5, 1, 9]), the 1 x 32 x 32768 paged causal prefill over 128 shuffled pages
    of 256, and grouped-query decode (64 query heads over 8 kv heads).  Each
    leg carries its own clocks and, on request, the oracle on a bounded sample
    of the same inputs."""
    import torch

    from paged_kv_cache_exact_b200 import accounting, api
    from paged_kv_cache_exact_b200.workloads import workload
    legs = {}

    def paged_inputs(w):
        t = [x.to(device) for x in (w.q, w.k_pages, w.v_pages, w.block_table, w.seq_lens)]
        out = torch.empty_like(t[0])
        ws = api.workspace_for(w.num_seqs, w.q.shape[1], 128, w.max_seq_len, w.page_size, device)
        fn = lambda: api.paged(*t, w.page_size, True, w.scale, max_seq_len=w.max_seq_len,
                               out=out, workspace=ws, stream=stream)
        return t, fn

    for name, w, desc in (
            ("decode_cfg4", workload(4), "paged decode, 16 seqs x 32 heads, d=128 bf16, "
             "seq_lens U[600,32768], page_size 256, seq 0 = 600 tokens on pages [5,1,9]"),
            ("decode_gqa", gqa_decode_workload(), "paged decode, 64 seqs x 64 query heads over "
             "8 kv heads, d=128 bf16, seq_lens U[512,8192], page_size 16")):
        t, fn = paged_inputs(w)
        ms, iters, clocks = _timed_leg(fn, stream, device)
        H, H_kv = w.q.shape[1], w.k_pages.shape[2]
        nbytes = accounting.decode_bytes(w.seq_lens.tolist(), H, H_kv, 128,
                                         max_pages=w.block_table.shape[1])
        gbs = nbytes / (ms / 1e3) / 1e9
        leg = {"workload": desc, "ms": ms, "calls": iters, "kv_gbs": gbs,
               "frac": gbs / peaks["hbm_gbs"], "bytes": nbytes,
               "sum_seq_lens": int(w.seq_lens.sum()), "clocks": clocks,
               "l2": f"KV pool {t[1].numel() * 4 / 1e9:.2f} GB > L2"}
        if cpu:
            leg["cpu_baseline"] = oracle_decode_sample(w)
        legs[name] = leg
        del t, fn

    w = workload(5)
    t, fn = paged_inputs(w)
    ms, iters, clocks = _timed_leg(fn, stream, device)
    flops = accounting.prefill_flops(1, 32, 32768, 32768, 128, True)
    tf = flops / (ms / 1e3) / 1e12
    tpeak, tsrc = tensor_peak(peaks, ms * iters / 1e3)
    leg = {"workload": "paged causal prefill 1x32x32768 d=128 bf16, 128 shuffled pages of 256 "
                       "(pool of 256 pages, the rest NaN-poisoned)",
           "ms": ms, "calls": iters, "tflops": tf, "frac": tf / peaks["bf16_tflops"],
           "frac_of_peak_used": tf / tpeak, "peak_source": tsrc, "flops": flops,
           "clocks": clocks}
    if cpu:
        leg["cpu_baseline"] = oracle_long_prefill_sample(w)
    legs["paged_prefill_cfg5"] = leg
    return legs


def measure_append(device, stream, peaks, iters=50):
    import torch

    run, moved, desc = append_setup(device)
    for _ in range(3):
        run(stream)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(device)
    e0.record(stream)
    for _ in range(iters):
        run(stream)
    e1.record(stream)
    torch.cuda.synchronize(device)
    ms = e0.elapsed_time(e1) / iters
    gbs = moved / (ms / 1e3) / 1e9
    return {"workload": desc, "ms": ms, "gbs": gbs, "frac": gbs / peaks["hbm_gbs"],
            "bytes": moved, "note": "paged_kv_append timed alone after the step loop; not in value"}


# ---------------------------------------------------------------------------
# the oracle on the host cores
# ---------------------------------------------------------------------------

def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


class OracleSample:
    """Bounded samples of the same workloads for the fp64 oracle."""

    def __init__(self, pre=None, dec=None):
        import numpy as np

        from paged_kv_cache_exact_b200.workloads import workload
        pre = workload(2) if pre is None else pre
        dec = workload(3) if dec is None else dec
        self.np = np
        self.Q = pre.Q.view(__import__("torch").int16).numpy()
        self.K = pre.K.view(__import__("torch").int16).numpy()
        self.V = pre.V.view(__import__("torch").int16).numpy()
        self.scale = pre.scale
        self.q = dec.q.view(__import__("torch").int16).numpy()
        self.kp = dec.k_pages.view(__import__("torch").int16).numpy()
        self.vp = dec.v_pages.view(__import__("torch").int16).numpy()
        self.table = dec.block_table.numpy()
        self.lens = dec.seq_lens.numpy()
        self.dscale = dec.scale

    def run(self, heads, rows, seq_heads):
        """Oracle over prefill (b, h) heads x rows and decode (seq, head) pairs;
        returns (prefill FLOPs, decode bytes) of the sample."""
        import oracle
        flops = 0
        for b, h in heads:
            oracle.attention_ref(self.Q[b, h], self.K[b, h], self.V[b, h], True, self.scale,
                                 rows=rows)
            flops += 4 * 128 * int(sum(r + 1 for r in rows))
        dbytes = 0
        for s, h in seq_heads:
            oracle.paged_attention_ref(self.q[s:s + 1, h:h + 1], self.kp[:, :, h:h + 1],
                                       self.vp[:, :, h:h + 1], self.table[s:s + 1],
                                       self.lens[s:s + 1], 16, True, self.dscale)
            dbytes += int(self.lens[s]) * 128 * 2 * 2
        return flops, dbytes


def oracle_decode_sample(w, budget_s=3.0):
    """The oracle on (sequence, query head) pairs of a decode workload, for
    about `budget_s` seconds, in the same unit as the GPU leg (GB/s of K/V;
    with grouped heads each query head counts its share of its kv head's
    rows, so the bytes of a whole group are counted once)."""
    import oracle
    import torch
    q = w.q.view(torch.int16).numpy()
    kp, vp = w.k_pages.view(torch.int16).numpy(), w.v_pages.view(torch.int16).numpy()
    table, lens = w.block_table.numpy(), w.seq_lens.numpy()
    S, H, H_kv = q.shape[0], q.shape[1], kp.shape[2]
    group = H // H_kv
    nbytes = pairs = 0
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < budget_s and pairs < S * H:
        s, h = pairs % S, (pairs // S) % H
        kvh = h // group
        oracle.paged_attention_ref(q[s:s + 1, h:h + 1], kp[:, :, kvh:kvh + 1],
                                   vp[:, :, kvh:kvh + 1], table[s:s + 1], lens[s:s + 1],
                                   w.page_size, True, w.scale)
        nbytes += int(lens[s]) * 128 * 2 * 2 / group   # this head's share of its kv head's rows
        pairs += 1
    dt = time.perf_counter() - t0
    return {"value": nbytes / dt / 1e9, "unit": "GB/s of K/V", "cores": _blas_threads(),
            "kind": "oracle", "sample": f"fp64 NumPy oracle on {pairs} (sequence, query head) "
                                        f"pairs of the same inputs, {dt:.1f} s"}


def oracle_long_prefill_sample(w, rows=512):
    """The oracle on every head of the long paged prefill at `rows` fixed query
    rows (the parity test's row mix), and a labelled linear extrapolation to
    all 32768 rows (the oracle forms each sampled row's scores against all
    keys, so its cost per row does not depend on the row)."""
    import numpy as np

    import oracle
    import torch
    rng = np.random.default_rng(5)
    fixed = {0, 1, 127, 128, 255, 256, 257, 16383, 32766, 32767}
    rest = [int(r) for r in rng.permutation(32768) if int(r) not in fixed][:rows - len(fixed)]
    sel = np.array(sorted(fixed | set(rest)))
    q = w.q.view(torch.int16).numpy()
    kp, vp = w.k_pages.view(torch.int16).numpy(), w.v_pages.view(torch.int16).numpy()
    table, lens = w.block_table.numpy(), w.seq_lens.numpy()
    t0 = time.perf_counter()
    for h in range(q.shape[1]):                  # one head at a time: bounded host memory
        oracle.paged_attention_ref(q[:, h:h + 1], kp[:, :, h:h + 1], vp[:, :, h:h + 1], table,
                                   lens, w.page_size, True, w.scale, rows=sel)
    dt = time.perf_counter() - t0
    flops = 4 * 128 * 32 * int(sum(int(r) + 1 for r in sel))     # visible pairs of the sample
    full_s = dt * 32768 / len(sel)
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s (visible pairs)",
            "cores": _blas_threads(), "kind": "oracle",
            "sample": f"fp64 NumPy oracle, all 32 heads x {len(sel)} fixed query rows of the same "
                      f"inputs, {dt:.1f} s",
            "extrapolated_full_s": full_s,
            "extrapolation": f"linear in rows: {dt:.1f} s x 32768 / {len(sel)} = {full_s:.0f} s "
                             "for the whole prefill (label: extrapolated, not run)"}


def cpu_baseline(peaks, budget_s=12.0, pre=None, dec=None):
    """The oracle as it stands, on rank 0's host cores, for about `budget_s`."""
    smp = OracleSample(pre, dec)
    np = smp.np
    rows = np.arange(0, 4096, 8)                   # every 8th row: the average causal row
    flops = dbytes = 0
    t0 = time.perf_counter()
    n_heads = n_pairs = 0
    while time.perf_counter() - t0 < budget_s and n_heads < 128:
        f, b = smp.run([(n_heads // 32, n_heads % 32)], rows, [(n_pairs // 32, n_pairs % 32)])
        flops, dbytes = flops + f, dbytes + b
        n_heads += 1
        n_pairs += 1
    dt = time.perf_counter() - t0
    return {"value": roofline_value(flops, dbytes, dt, peaks), "unit": UNIT,
            "cores": _blas_threads(), "kind": "oracle",
            "sample": f"fp64 NumPy oracle: {n_heads} prefill heads x {len(rows)} rows (every 8th) "
                      f"+ {n_pairs} decode (seq, head) pairs of the same workloads, {dt:.1f} s",
            "prefill_gflops": flops / dt / 1e9, "decode_gbs": dbytes / dt / 1e9}


def run_reference(args):
    """Reference arm: the fp64 oracle on the host cores, one bounded sample per step."""
    peaks, _ = load_peaks()
    smp = OracleSample()
    np = smp.np
    rows = np.arange(0, 4096, 128)                 # 32 rows of one head per step
    for i in range(args.warmup):
        smp.run([(0, i % 32)], rows, [(i % 64, 0)])
    flops = dbytes = 0
    t0 = time.perf_counter()
    for k in range(args.steps):
        f, b = smp.run([((k // 32) % 4, k % 32)], rows, [(k % 64, (k // 64) % 32)])
        flops, dbytes = flops + f, dbytes + b
    dt = time.perf_counter() - t0
    value = roofline_value(flops, dbytes, dt, peaks)
    sample = ("fp64 NumPy oracle per step: 1 prefill head x 32 rows (every 128th) + "
              "1 decode (seq, head) pair of the same workloads")
    return {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (same seeded workloads)", "impl": "reference",
            "config": {"workload": WORKLOAD, "parallelism": "host cores (rank 0)"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": _blas_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


# ---------------------------------------------------------------------------
# profiling cases: one kernel family on a small case, for ncu captures
# ---------------------------------------------------------------------------

PROFILE_CASES = {
    "step": "the serving step: causal prefill B=4 H=32 N=4096 d=128 + paged decode 64 seqs x 32 "
            "heads, seq_lens U[512,8192], page_size 16 (the bench's timed step, 3 launches/iter)",
    "prefill": "causal prefill B=4 H=32 N=4096 d=128 (the step's prefill, 1 launch/iter)",
    "prefill-fp8": "causal prefill B=4 H=32 N=4096 d=128, e4m3 Q/K with per-tensor scales, "
                   "bf16 V/O",
    "paged-prefill": "paged causal prefill 1x32x32768x128, 128 shuffled pages of 256",
    "decode16": "paged decode, 16 seqs x 32 heads, seq_lens U[512,8192], page_size 16 "
                "(the step's decode distribution, a quarter of the sequences)",
    "append": "paged KV append, 64 seqs x 512 new tokens, H_kv=32 d=128 bf16, page 16",
    "decode-gqa": "paged decode with grouped heads, 64 seqs x 64 query heads over 8 kv heads, "
                  "seq_lens U[512,8192], page_size 16",
    "decode256": "paged decode, 16 seqs x 32 heads, seq_lens U[600,32768], page_size 256, "
                 "seq 0 = 600 tokens on pages [5,1,9]",
}


def run_profile(args):
    import torch

    from paged_kv_cache_exact_b200 import api
    from paged_kv_cache_exact_b200.workloads import make_paged, workload
    dev = torch.device("cuda", 0)
    if args.profile == "step":
        torch.cuda.set_device(dev)
        prefill, decode, _, _, meta = build_step(dev)
        stream = torch.cuda.current_stream(dev)
        for _ in range(args.steps):
            prefill(stream)
            decode(stream)
        torch.cuda.synchronize(dev)
        print(json.dumps({"profile": "step", "case": PROFILE_CASES["step"],
                          "iterations": args.steps,
                          "launches_per_step": meta["launches_per_step"]}))
        return
    if args.profile == "append":
        run, moved, desc = append_setup(dev)
        for _ in range(args.steps):
            run(None)
        torch.cuda.synchronize(dev)
        print(json.dumps({"profile": "append", "case": desc, "iterations": args.steps,
                          "bytes_per_launch": moved}))
        return
    if args.profile == "prefill":
        w = workload(2)
        Q, K, V = w.Q.to(dev), w.K.to(dev), w.V.to(dev)
        O = torch.empty_like(Q)
        fn = lambda: api.prefill(Q, K, V, True, w.scale, out=O)
    elif args.profile == "prefill-fp8":
        from paged_kv_cache_exact_b200 import binding as B
        w = workload(2)
        Q, K, V = w.Q.to(dev), w.K.to(dev), w.V.to(dev)
        qd = float(Q.float().abs().max()) / 448.0
        kd = float(K.float().abs().max()) / 448.0
        Q8 = (Q.float() / qd).to(torch.float8_e4m3fn).view(torch.uint8)
        K8 = (K.float() / kd).to(torch.float8_e4m3fn).view(torch.uint8)
        O = torch.empty_like(V)
        Bn, H, N, d = Q.shape
        fn = lambda: B.attn_prefill_fp8qk(Q8, K8, V, O, Bn, H, N, d, True, w.scale, qd, kd)
    else:
        if args.profile == "paged-prefill":
            w = workload(5)
        elif args.profile == "decode256":
            w = workload(4)
        elif args.profile == "decode-gqa":
            w = gqa_decode_workload()
        else:
            w = make_paged(1003, (512, 8192, 16), 32, 128, 16, q_len=1, decoys=16)
        t = [x.to(dev) for x in (w.q, w.k_pages, w.v_pages, w.block_table, w.seq_lens)]
        O = torch.empty_like(t[0])
        ws = api.workspace_for(w.num_seqs, w.q.shape[1], 128, w.max_seq_len, w.page_size, dev)
        fn = lambda: api.paged(*t, w.page_size, True, w.scale, max_seq_len=w.max_seq_len,
                               out=O, workspace=ws)
    for _ in range(args.steps):
        fn()
    torch.cuda.synchronize(dev)
    units = (int(w.seq_lens.sum()) * w.k_pages.shape[2]
             if args.profile in ("decode16", "decode-gqa", "decode256") else None)
    print(json.dumps({"profile": args.profile, "case": PROFILE_CASES[args.profile],
                      "iterations": args.steps, "decode_units": units}))


# ---------------------------------------------------------------------------

def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile", choices=sorted(PROFILE_CASES),
                    help="run one kernel family --steps times on a small case (for ncu) and exit")
    args = ap.parse_args(argv)
    if args.profile:
        run_profile(args)
        return 0
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(format_line(run_reference(args)), flush=True)
        return 0

    dist = None
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist_mod
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        dist_mod.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))
        dist = dist_mod
    try:
        line, (pre, dec) = run_gpu(args, rank, world, dist)
        if rank == 0:
            if world == 1 and not args.no_cpu_baseline:
                line["cpu_baseline"] = cpu_baseline(load_peaks()[0], pre=pre, dec=dec)
            print(format_line(line), flush=True)
    finally:
        if dist is not None:
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
