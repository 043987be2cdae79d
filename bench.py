#!/usr/bin/env python
"""Bench: skip-softmax sparse attention forward on B200.

Default workload: the Llama-3.1-8B-shaped prefill (B=1, Hq=32, Hkv=8,
L=8192, d=128, causal, Br=Bc=128, skip-softmax lambda=1e-3), seeded
synthetic bf16 Q/K/V.  One step = one ssa_fwd launch over that batch.

Prints ONE JSON line.  ``value`` is the dense-equivalent attention TFLOP/s
(4 d B Hq x visible pairs / time) summed over ranks; the same line carries
executed TFLOP/s (2 Br Bc d x (visited + kept tiles) / time), the fraction of
visited tiles skipped, tokens/s, the roofline of the kernel, an end-to-end
figure through the C ABI with host buffers, and the CPU oracle's throughput on
a bounded sample of the same workload.

Multi-GPU: one process per GPU (torchrun); the path has no exchange step, so
each rank runs its own replica of the workload (weak scaling) and time is the
max over ranks.  ``--impl reference`` times the CPU oracle instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import select
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from softmax_ssa_fwd_b200.inputs import MODE_NM, MODE_SKIP, WORKLOADS, make_inputs  # noqa: E402

KERNEL_SRC = [os.path.join(ROOT, "softmax_ssa_fwd_b200", "csrc", f) for f in ("ssa_fwd.cu", "ptx.cuh")]
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "ssa_fwd_traffic.json")  # ncu DRAM bytes, keyed by kernel source hash


def kernel_hash() -> str:
    h = hashlib.sha256()
    for f in KERNEL_SRC:
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d["bf16_tflops"], d.get("bf16_tflops_sustained"), d["hbm_gbs"], "measured"
    return 1590.0, 1400.0, 6650.0, "fallback"


def dense_equiv_flops(w, Lq=None) -> float:
    Lq = Lq or w.L
    Lk = w.L
    if w.causal:
        off = Lk - Lq
        i = np.arange(Lq, dtype=np.int64)
        pairs = int(np.clip(i + off + 1, 0, Lk).sum())
    else:
        pairs = Lq * Lk
    return 4.0 * w.d * w.B * w.Hq * pairs


def reduce_max(x: float, dist, device) -> float:
    """Max over ranks (the job's time is its slowest rank's); identity without a group."""
    if dist is None:
        return x
    t = torch.tensor([x], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_rank: float, world: int, ms_max: float) -> float:
    """Whole-job throughput: every rank processes its own replica of the workload."""
    return world * units_per_rank / (ms_max * 1e-3)


def workload_name(w, lam):
    s = (f"{w.name}: B={w.B} Hq={w.Hq} Hkv={w.Hkv} L={w.L} d={w.d} "
         f"{'causal' if w.causal else 'non-causal'} Br={w.Br} Bc={w.Bc}")
    if w.mode & MODE_SKIP:
        s += f" skip lambda={lam:g}"
    if w.mode & MODE_NM:
        s += f" N:M {w.n}:{w.m} sink={w.sink} recent={w.recent}"
    if w.sink_coef not in (0.0, 3.0) or w.local_alpha:
        s += f" (stress: sink_coef={w.sink_coef:g} local_alpha={w.local_alpha:g})"
    return s


class Clocks:
    """nvidia-smi sampler running during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, local_rank: int):
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        ids = [x for x in vis.split(",") if x.strip()] if vis else []
        self.idx = ids[local_rank].strip() if local_rank < len(ids) else local_rank
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return self
        # nvidia-smi's start-up can hold the driver for seconds; the timed
        # region starts only after its first sample has arrived.
        self.first = ""
        ready, _, _ = select.select([self.proc.stdout], [], [], 20.0)
        if ready:
            self.first = self.proc.stdout.readline()
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                rest, _ = self.proc.communicate(timeout=5)
                self.out = self.first + rest
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out = ""

    def summary(self):
        rows_by_gpu = {}
        for line in self.out.splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows_by_gpu.setdefault(parts[0], []).append((float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        rows = rows_by_gpu.get(str(self.idx))
        if rows is None and len(rows_by_gpu) == 1:
            rows = next(iter(rows_by_gpu.values()))
        rows = rows or []
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        maxmhz = max(r[1] for r in rows)
        loaded = [r for r in rows if r[0] > 0.3 * maxmhz] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in loaded for i, v in enumerate(r[2]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": maxmhz,
                "reasons": reasons, "samples": len(loaded)}


_CPU_INPUTS = {}


def cpu_baseline(w, lam, budget_s: float, seed: int = 7):
    """Time the fp64 oracle on a bounded random sample of work items of the
    same workload (inputs generated on the CPU with the same recipe)."""
    from oracle import run_items
    g = torch.Generator().manual_seed(seed)
    if w not in _CPU_INPUTS:
        _CPU_INPUTS[w] = make_inputs(w, "cpu")
    q, k, v = _CPU_INPUTS[w]
    cores = len(os.sched_getaffinity(0))
    nQ = -(-w.L // w.Br)
    done_items, flops, t_total = 0, 0.0, 0.0
    while done_items == 0 or t_total < budget_s:
        n = cores
        items = [(int(torch.randint(w.B, (1,), generator=g)), int(torch.randint(w.Hq, (1,), generator=g)),
                  int(torch.randint(nQ, (1,), generator=g))) for _ in range(n)]
        t0 = time.perf_counter()
        run_items(q, k, v, causal=w.causal, scale=w.scale, mode=w.mode, lam=lam, n=w.n, m=w.m,
                  sink=w.sink, recent=w.recent, Br=w.Br, Bc=w.Bc, items=items, nthreads=cores)
        t_total += time.perf_counter() - t0
        for (_, _, t) in items:
            r0, r1 = t * w.Br, min(w.L, t * w.Br + w.Br)
            if w.causal:
                flops += 4.0 * w.d * sum(min(i + 1, w.L) for i in range(r0, r1))
            else:
                flops += 4.0 * w.d * (r1 - r0) * w.L
        done_items += n
    return {"value": flops / t_total / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"{done_items} random (b, head, q-tile) work items of {w.name} (lambda={lam:g}), "
                      f"fp64 C oracle, {t_total:.1f} s wall; dense-equivalent FLOPs of the sample / wall"}


def run_reference(args, w, lam, rank, world):
    if rank != 0:
        return 0
    # each step: one batch of work items (one per host core) of the workload
    per_step = []
    info = None
    for s in range(min(args.warmup, 1)):
        (decode_cpu_baseline if w.Lq else cpu_baseline)(w, lam, 0.0, seed=99)
    for s in range(max(1, args.steps)):
        info = (decode_cpu_baseline(w, lam, 0.0, seed=100 + s) if w.Lq
                else cpu_baseline(w, lam, 0.0, seed=100 + s))
        per_step.append(info["value"])
    val = statistics.median(per_step)
    metric = "attn decode HBM GB/s (K, V, Q, O, lse once)" if w.Lq else "attn fwd TFLOP/s (dense-equiv)"
    line = {"impl": "reference", "metric": metric, "value": val,
            "unit": info["unit"], "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": workload_name(w, lam)},
            "cpu_baseline": dict(info, value=val),
            "e2e": {"value": val, "unit": info["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def block_mask_bits(w, density: float, seed: int) -> np.ndarray:
    """Seeded random key-block selection [B, Hkv, nQ, nK] (bool) restricted to the
    visible tiles; key tile 0 and each query block's last visible tile are always
    selected."""
    nQ, nK = -(-w.L // w.Br), -(-w.L // w.Bc)
    rng = np.random.default_rng(seed)
    bits = rng.random((w.B, w.Hkv, nQ, nK)) < density
    for qt in range(nQ):
        last = min(nK - 1, (min(w.L, qt * w.Br + w.Br) - 1) // w.Bc) if w.causal else nK - 1
        bits[:, :, qt, last + 1:] = False
        bits[:, :, qt, 0] = True
        bits[:, :, qt, last] = True
    return bits


def pack_bits(bits: np.ndarray) -> np.ndarray:
    """[..., nK] bool -> [..., ceil(nK / 32)] uint32, bit kt % 32 of word kt // 32."""
    nK = bits.shape[-1]
    nKw = -(-nK // 32)
    padded = np.zeros(bits.shape[:-1] + (nKw * 32,), dtype=np.uint32)
    padded[..., :nK] = bits
    words = np.zeros(bits.shape[:-1] + (nKw,), dtype=np.uint32)
    for i in range(32):
        words |= padded[..., i::32] << np.uint32(i)
    return words


# Every workload of the method's targets, measured on the same device in the
# same run as the headline (each its own line in the JSON "configs" object):
# the literal workloads, the two labelled stress variants that make the skip
# path run, the decode path and the bitmap-selected path.
SWEEP = [
    ("tiny lambda=0", "tiny", 0.0, {}),
    ("tiny lambda=1e-3", "tiny", 1e-3, {}),
    ("tiny lambda=1e-2", "tiny", 1e-2, {}),
    ("llama8k lambda=1e-4", "llama8k", 1e-4, {}),
    ("llama8k lambda=1e-3", "llama8k", 1e-3, {}),
    ("llama8k lambda=1e-2", "llama8k", 1e-2, {}),
    ("llama4k_nm24", "llama4k_nm24", 0.0, {}),
    ("llama4k_nm48", "llama4k_nm48", 0.0, {}),
    ("wan lambda=1e-3", "wan", 1e-3, {}),
    ("qwen32k skip+2:4 lambda=1e-3", "qwen32k", 1e-3, {}),
    ("stress llama8k sink_coef=12 lambda=1e-3", "llama8k", 1e-3, {"sink_coef": 12.0}),
    ("stress wan local_alpha=2.5 lambda=1e-3", "wan", 1e-3, {"local_alpha": 2.5}),
    ("llama8k key blocks by bitmap density 0.25 lambda=1e-3", "llama8k", 1e-3, {"mask_density": 0.25}),
    ("decode qwen32k_decode lambda=1e-4", "qwen32k_decode", 1e-4, {}),
    ("sol_proxy 84/512 exact blocks, proxy off", "sol_proxy", 0.0, {"exact_blocks": 84}),
    ("sol_proxy 84/512 exact blocks, proxy on", "sol_proxy", 0.0, {"exact_blocks": 84, "proxy": True}),
]


def exact_block_bits(w, per_row: int, seed: int) -> np.ndarray:
    """Seeded selection of exactly per_row key blocks for every (batch, KV
    head, query block): [B, Hkv, nQ, nK] bool."""
    nQ, nK = -(-w.L // w.Br), -(-w.L // w.Bc)
    rng = np.random.default_rng(seed)
    bits = np.zeros((w.B, w.Hkv, nQ, nK), bool)
    for b in range(w.B):
        for h in range(w.Hkv):
            for qt in range(nQ):
                bits[b, h, qt, rng.choice(nK, size=per_row, replace=False)] = True
    return bits


def block_summaries_dev(k, v, Bc: int):
    """The caller's proxy summaries on the device (input preparation, not
    timed): per key block the mean of its keys and the sum of its values, bf16."""
    B, L, H, d = k.shape
    nK = -(-L // Bc)
    pad = nK * Bc - L
    kf = torch.nn.functional.pad(k.float(), (0, 0, 0, 0, 0, pad)).view(B, nK, Bc, H, d)
    vf = torch.nn.functional.pad(v.float(), (0, 0, 0, 0, 0, pad)).view(B, nK, Bc, H, d)
    cnt = torch.full((nK,), float(Bc), device=k.device)
    cnt[-1] = Bc - pad
    km = (kf.sum(dim=2) / cnt[None, :, None, None]).to(torch.bfloat16).contiguous()
    vs = vf.sum(dim=2).to(torch.bfloat16).contiguous()
    return km, vs


def sweep_configs(dev, stream, target_ms: float = 400.0):
    """Time every SWEEP entry on this GPU: CUDA events on the launching
    stream, 2 warm-up launches, then enough launches for ~target_ms (at least
    3).  Workloads smaller than L2 alternate two input sets."""
    from softmax_ssa_fwd_b200 import ssa
    bf16_peak, _, hbm_peak, src = peaks()
    res = {}
    for label, name, lam, extra in SWEEP:
        w = WORKLOADS[name]
        dens = extra.get("mask_density", 0.0)
        exact = extra.get("exact_blocks", 0)
        proxy = extra.get("proxy", False)
        kw = {k_: v_ for k_, v_ in extra.items() if k_ not in ("mask_density", "exact_blocks", "proxy")}
        if kw:
            w = w.with_(**kw)
        if w.Lq:  # decode
            nsets = 2
            ws_bytes = ssa.ssa_decode_workspace_bytes(w.B, w.Hq, w.Lq, w.d, w.splits)
            sets = []
            for si in range(nsets):
                q, k, v = make_inputs(w.with_(seed=w.seed + 1000 * si), dev)
                sets.append((q, k, v, torch.empty_like(q),
                             torch.empty(w.B, w.Hq, w.Lq, dtype=torch.float32, device=dev),
                             torch.empty(w.B, w.Hq, dtype=torch.int32, device=dev),
                             torch.empty(ws_bytes, dtype=torch.uint8, device=dev)))

            def launch(i):
                q, k, v, o, l_, c, ws = sets[i % nsets]
                return ssa.ssa_decode(q, k, v, o, l_, c, w.B, w.Hq, w.Hkv, w.Lq, w.L, w.d, w.causal, w.scale,
                                      lam, w.Bc, w.splits, ws, ws_bytes, stream)
        else:
            in_bytes = 2 * (w.B * w.L * w.Hq * w.d + 2 * w.B * w.L * w.Hkv * w.d)
            nsets = 2 if in_bytes < 256e6 else 1
            sets = []
            for si in range(nsets):
                q, k, v = make_inputs(w.with_(seed=w.seed + 1000 * si), dev)
                sets.append((q, k, v, torch.empty_like(q),
                             torch.empty(w.B, w.Hq, w.L, dtype=torch.float32, device=dev),
                             torch.empty(w.B, w.Hq, -(-w.L // w.Br), dtype=torch.int32, device=dev)))
            mask_bits = mask_dev = None
            if dens > 0:
                mask_bits = block_mask_bits(w, dens, seed=w.seed)
            if exact > 0:
                mask_bits = exact_block_bits(w, exact, seed=w.seed)
            if mask_bits is not None:
                mask_dev = torch.from_numpy(pack_bits(mask_bits).view(np.int32)).to(dev)
            summ = [block_summaries_dev(s_[1], s_[2], w.Bc) for s_ in sets] if proxy else None

            def launch(i):
                q, k, v, o, l_, c = sets[i % nsets]
                if proxy:
                    km, vs = summ[i % nsets]
                    return ssa.ssa_fwd_blockmask_proxy(q, k, v, o, l_, w.B, w.Hq, w.Hkv, w.L, w.L, w.d, w.scale,
                                                       w.Br, w.Bc, mask_dev, km, vs, stream)
                if mask_dev is not None:
                    return ssa.ssa_fwd_blockmask(q, k, v, o, l_, c, w.B, w.Hq, w.Hkv, w.L, w.L, w.d, w.causal,
                                                 w.scale, w.mode, lam, w.n, w.m, w.sink, w.recent, w.Br, w.Bc,
                                                 mask_dev, stream)
                return ssa.ssa_fwd(q, k, v, o, l_, c, w.B, w.Hq, w.Hkv, w.L, w.L, w.d, w.causal, w.scale,
                                   w.mode, lam, w.n, w.m, w.sink, w.recent, w.Br, w.Bc, stream)

        for i in range(2):
            if launch(i) != 0:
                raise RuntimeError(f"{label}: launch refused")
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        launch(0)
        e1.record(stream)
        e1.synchronize()
        steps = max(3, min(500, int(target_ms / max(e0.elapsed_time(e1), 1e-3))))
        torch.cuda.synchronize()
        e0.record(stream)
        for i in range(steps):
            launch(i)
        e1.record(stream)
        e1.synchronize()
        ms = e0.elapsed_time(e1) / steps
        if ssa.ssa_device_status(stream) != 0:
            raise RuntimeError(f"{label}: device-side timeout")
        entry = {"workload": workload_name(w, lam), "ms_per_step": ms, "steps": steps}
        if w.Lq:
            nK = -(-w.L // w.Bc)
            skipped = sum(float(s_[5].sum().item()) for s_ in sets) / nsets
            visited = float(w.B * w.Hq * nK)
            gbs = decode_alg_bytes(w) / (ms * 1e-3) / 1e9
            entry.update({"hbm_gbs": gbs, "hbm_frac_of_peak": gbs / hbm_peak,
                          "dense_equiv_tflops": dense_equiv_flops(w, Lq=w.Lq) / (ms * 1e-3) / 1e12,
                          "tiles_skipped_frac": skipped / visited,
                          "tokens_per_s": w.B * w.Lq / (ms * 1e-3)})
        elif exact > 0:
            # algorithmic work: the exact blocks (QK^T and P.V of Br x Bc x d each),
            # plus, with proxies, one score and one P.V term of d per row and omitted block
            nQ, nK = -(-w.L // w.Br), -(-w.L // w.Bc)
            sel = float(mask_bits.sum()) * (w.Hq // w.Hkv)
            fl = 4.0 * w.Br * w.Bc * w.d * sel
            if proxy:
                fl += 4.0 * w.d * w.B * w.Hq * w.L * (nK - exact)
            entry.update({"algorithmic_tflops": fl / (ms * 1e-3) / 1e12,
                          "algorithmic_frac_of_peak": fl / (ms * 1e-3) / 1e12 / bf16_peak,
                          "tiles_skipped_frac": 0.0,
                          "page_b200_ms": 1.2121 if proxy else 1.1261,
                          "page_b200_ms_note": "the page's attention kernel p50 on its own B200 and data "
                                               "(context, not the same inputs)"})
        else:
            visited = ssa.ssa_visited_tiles(w.causal, w.L, w.L, w.Br, w.Bc) * w.B * w.Hq
            if mask_bits is not None:
                visited = int(mask_bits.sum()) * (w.Hq // w.Hkv)
            skipped = sum(float(s_[5].sum().item()) for s_ in sets) / nsets
            kept = visited - skipped
            fd = dense_equiv_flops(w) / (ms * 1e-3) / 1e12
            fe = 2.0 * w.Br * w.Bc * w.d * (visited + kept) / (ms * 1e-3) / 1e12
            entry.update({"dense_equiv_tflops": fd, "executed_tflops": fe,
                          "executed_frac_of_peak": fe / bf16_peak, "dense_equiv_frac_of_peak": fd / bf16_peak,
                          "tiles_skipped_frac": skipped / visited, "tiles_visited": visited,
                          "tokens_per_s": w.B * w.L / (ms * 1e-3)})
        res[label] = entry
        del sets
        torch.cuda.empty_cache()
    res["_peak"] = {"bf16_tflops": bf16_peak, "hbm_gbs": hbm_peak, "source": f"{src} (burst)"}
    return res


def decode_cpu_baseline(w, lam, budget_s: float, seed: int = 7):
    """The fp64 decode oracle (numpy) on a bounded sample of (sequence, head)
    pairs of the decode workload; dense-equivalent FLOPs of the sample / wall."""
    from oracle.decode import decode as decode_oracle
    q, k, v = make_inputs(w, "cpu")
    g = torch.Generator().manual_seed(seed)
    done, t_total = 0, 0.0
    while done == 0 or t_total < budget_s:
        heads = [(int(torch.randint(w.B, (1,), generator=g)), int(torch.randint(w.Hq, (1,), generator=g)))]
        t0 = time.perf_counter()
        decode_oracle(q, k, v, causal=w.causal, scale=w.scale, lam=lam, Bc=w.Bc, num_splits=w.splits,
                      heads=heads)
        t_total += time.perf_counter() - t0
        done += 1
    per_head = decode_alg_bytes(w) / (w.B * w.Hq)
    return {"value": per_head * done / t_total / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"{done} random (sequence, head) pairs of {w.name} (lambda={lam:g}), fp64 numpy "
                      f"decode oracle, {t_total:.1f} s wall; the pairs' share of the algorithmic bytes / wall"}


def decode_alg_bytes(w) -> float:
    """K and V read once, Q and O (bf16) and lse (fp32) once."""
    return 2.0 * w.B * w.L * w.Hkv * w.d * 2 + 2.0 * 2 * w.B * w.Lq * w.Hq * w.d + 4.0 * w.B * w.Hq * w.Lq


def run_decode(args, w, lam, rank, world, local_rank):
    """Decode leg: ssa_decode on a resident KV cache.  HBM-bound, so the
    roofline is bytes: K and V read once, Q, O and lse once."""
    import torch.distributed as tdist
    dist = None
    if world > 1:
        import datetime
        dist = tdist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    from softmax_ssa_fwd_b200 import ssa
    dev = torch.device("cuda", local_rank)
    nK = -(-w.L // w.Bc)
    ws_bytes = ssa.ssa_decode_workspace_bytes(w.B, w.Hq, w.Lq, w.d, w.splits)
    sets = []
    for s in range(2):  # two KV caches of 1.07 GB each, alternated: > 126 MB L2
        q, k, v = make_inputs(w.with_(seed=w.seed + 1000 * s + 17 * rank), dev)
        out = torch.empty_like(q)
        lse = torch.empty(w.B, w.Hq, w.Lq, dtype=torch.float32, device=dev)
        cnt = torch.empty(w.B, w.Hq, dtype=torch.int32, device=dev)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
        sets.append((q, k, v, out, lse, cnt, ws))
    stream = torch.cuda.current_stream(dev)

    def step(i, qq=None):
        q, k, v, out, lse, cnt, ws = sets[i & 1]
        st = ssa.ssa_decode(q if qq is None else qq, k, v, out, lse, cnt, w.B, w.Hq, w.Hkv, w.Lq, w.L,
                            w.d, w.causal, w.scale, lam, w.Bc, w.splits, ws, ws_bytes, stream)
        if st != 0:
            raise RuntimeError(ssa.status_string(st))

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with Clocks(local_rank) as clk:
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        for i in range(args.steps):
            step(i)
        e1.record(stream)
        e1.synchronize()
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
    ms_step = reduce_max(e0.elapsed_time(e1), dist, dev) / args.steps
    skipped = float(sets[(args.steps - 1) & 1][5].sum().item())
    visited = float(w.B * w.Hq * nK)
    bf16_peak, _, hbm_peak, src = peaks()
    alg_bytes = decode_alg_bytes(w)
    flops = dense_equiv_flops(w, Lq=w.Lq)
    gbs = job_rate(alg_bytes, world, ms_step) / 1e9
    # e2e: the step's new query rows from pinned host memory, out + lse + counts back
    e2e = None
    if not args.no_e2e:
        q, k, v, out, lse, cnt, ws = sets[0]
        hq_ = q.cpu().pin_memory()
        ho, hl, hc = (torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in (out, lse, cnt))
        dq = torch.empty_like(q)
        n_e2e = max(3, min(args.steps, 50))

        def e2e_step():
            dq.copy_(hq_, non_blocking=True)
            step(0, dq)
            ho.copy_(out, non_blocking=True)
            hl.copy_(lse, non_blocking=True)
            hc.copy_(cnt, non_blocking=True)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(n_e2e):
            e2e_step()
        e1.record(stream)
        e1.synchronize()
        ems = reduce_max(e0.elapsed_time(e1), dist, dev) / n_e2e
        e2e = {"value": job_rate(alg_bytes, world, ems) / 1e9, "unit": "GB/s",
               "h2d_bytes_per_step": hq_.numel() * hq_.element_size(),
               "d2h_bytes_per_step": sum(t.numel() * t.element_size() for t in (ho, hl, hc)),
               "ms_per_step": ems, "steps": n_e2e, "kv_cache": "resident on the GPU (decode state)"}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = decode_cpu_baseline(w, lam, args.cpu_budget)
    if rank == 0:
        line = {
            "metric": "attn decode HBM GB/s (K, V, Q, O, lse once)", "value": gbs, "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": workload_name(w, lam) + f" decode Lq={w.Lq} splits={w.splits}",
                       "parallelism": f"replicas x{world}",
                       "l2": "two KV caches of 1.07 GB alternated (> 126 MB L2)"},
            "dense_equiv_tflops": job_rate(flops, world, ms_step) / 1e12,
            "tiles_skipped_frac": skipped / visited, "tiles_visited": visited, "tiles_skipped": skipped,
            "tokens_per_s": job_rate(w.B * w.Lq, world, ms_step),
            "roofline": {"bound": "hbm", "achieved": gbs / world, "peak": hbm_peak, "unit": "GB/s",
                         "frac": gbs / world / hbm_peak, "traffic": None,
                         "peak_source": f"{src} HBM copy",
                         "kernel": "ssa_dec::decode_split_kernel + decode_combine_kernel",
                         "algorithmic_bytes": alg_bytes},
            "gpu_launches": 2 * args.steps,
            "clocks": clk.summary(), "e2e": e2e, "cpu_baseline": cpu, "kernel_hash": kernel_hash(),
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="llama8k", choices=sorted(WORKLOADS))
    ap.add_argument("--lam", type=float, default=None)
    ap.add_argument("--sink-coef", type=float, default=None)
    ap.add_argument("--local-alpha", type=float, default=None)
    ap.add_argument("--L", type=int, default=None, help="override the sequence length")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--splits", type=int, default=None, help="decode: override the key splits")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-workload sweep that fills the line's \"configs\" object")
    ap.add_argument("--mask-density", type=float, default=0.0,
                    help="select key blocks by a seeded random bitmap of this density "
                         "(ssa_fwd_blockmask); key tile 0 and the diagonal tile always selected")
    ap.add_argument("--exact-blocks", type=int, default=0,
                    help="select exactly this many key blocks per query block, seeded at random "
                         "(ssa_fwd_blockmask; the selection the sol_proxy workload is measured with)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3

    w = WORKLOADS[args.workload]
    if args.sink_coef is not None:
        w = w.with_(sink_coef=args.sink_coef)
    if args.local_alpha is not None:
        w = w.with_(local_alpha=args.local_alpha)
    if args.splits is not None:
        w = w.with_(splits=args.splits)
    if args.L is not None:
        if w.rope == "3d":
            raise SystemExit("--L does not apply to the 3D-rotary video workload")
        w = w.with_(L=args.L, name=f"{w.name}@L{args.L}")
    lam = args.lam if args.lam is not None else (w.lambdas[0] if w.Lq else (1e-3 if w.mode & MODE_SKIP else 0.0))

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        return run_reference(args, w, lam, rank, world)
    if w.Lq:
        torch.cuda.set_device(local_rank)
        return run_decode(args, w, lam, rank, world, local_rank)

    torch.cuda.set_device(local_rank)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    from softmax_ssa_fwd_b200 import ssa

    dev = torch.device("cuda", local_rank)
    # two input sets, alternated between steps (llama8k: 2 x 168 MB > 126 MB L2)
    set_mb = 2 * (w.B * w.L * w.Hq * w.d + 2 * w.B * w.L * w.Hkv * w.d) / 1e6
    sets = []
    for s in range(2):
        q, k, v = make_inputs(w.with_(seed=w.seed + 1000 * s + 17 * rank), dev)
        out = torch.empty_like(q)
        lse = torch.empty(w.B, w.Hq, w.L, dtype=torch.float32, device=dev)
        cnt = torch.empty(w.B, w.Hq, -(-w.L // w.Br), dtype=torch.int32, device=dev)
        sets.append((q, k, v, out, lse, cnt))
    stream = torch.cuda.current_stream(dev)
    nQ, nK = -(-w.L // w.Br), -(-w.L // w.Bc)
    mask_bits = mask_dev = None
    if args.mask_density > 0:
        mask_bits = block_mask_bits(w, args.mask_density, seed=w.seed + 31 * rank)
    if args.exact_blocks > 0:
        mask_bits = exact_block_bits(w, args.exact_blocks, seed=w.seed + 31 * rank)
    if mask_bits is not None:
        mask_dev = torch.from_numpy(pack_bits(mask_bits).view(np.int32)).to(dev)

    def fwd(q, k, v, out, lse, cnt):
        if mask_dev is not None:
            return ssa.ssa_fwd_blockmask(q, k, v, out, lse, cnt, w.B, w.Hq, w.Hkv, w.L, w.L, w.d, w.causal,
                                         w.scale, w.mode, lam, w.n, w.m, w.sink, w.recent, w.Br, w.Bc,
                                         mask_dev, stream)
        return ssa.ssa_fwd(q, k, v, out, lse, cnt, w.B, w.Hq, w.Hkv, w.L, w.L, w.d, w.causal, w.scale,
                           w.mode, lam, w.n, w.m, w.sink, w.recent, w.Br, w.Bc, stream)

    def step(i):
        st = fwd(*sets[i & 1])
        if st != 0:
            raise RuntimeError(ssa.status_string(st))

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    if ssa.ssa_device_status(stream) != 0:
        raise RuntimeError("device-side timeout during warm-up")

    def barrier():
        if dist is not None:
            dist.barrier()

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with Clocks(local_rank) as clk:
        barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        for i in range(args.steps):
            step(i)
        e1.record(stream)
        e1.synchronize()
        torch.cuda.synchronize()
        barrier()
    ms = e0.elapsed_time(e1)
    if ssa.ssa_device_status(stream) != 0:
        raise RuntimeError("device-side timeout in the timed region")
    ms = reduce_max(ms, dist, dev)
    ms_step = ms / args.steps

    # skip statistics of the timed workload (identical every step per input set)
    visited = ssa.ssa_visited_tiles(w.causal, w.L, w.L, w.Br, w.Bc) * w.B * w.Hq
    if mask_bits is not None:  # selected visible tiles, per KV head times its query heads
        visited = int(mask_bits.sum()) * (w.Hq // w.Hkv)
    skipped = sum(int(s[5].sum()) for s in sets) / len(sets)
    kept = visited - skipped
    flops_dense = dense_equiv_flops(w)
    flops_exec = 2.0 * w.Br * w.Bc * w.d * (visited + kept)
    tflops_dense = job_rate(flops_dense, world, ms_step) / 1e12
    tflops_exec = job_rate(flops_exec, world, ms_step) / 1e12
    bf16_peak, bf16_sus, hbm_peak, src = peaks()
    tokens = job_rate(w.B * w.L, world, ms_step)

    traffic = None
    if os.path.exists(TRAFFIC_FILE):
        with open(TRAFFIC_FILE) as f:
            tr = json.load(f)
        if tr.get("kernel_hash") == kernel_hash() and tr.get("workload") == w.name:
            traffic = tr.get("dram_bytes_per_launch")

    # end to end through the C ABI with host buffers: pinned host inputs ->
    # device, forward, out + lse + counts back to pinned host, every step
    e2e = None
    if not args.no_e2e:
        q, k, v, out, lse, cnt = sets[0]
        hq_, hk_, hv_ = (t.cpu().pin_memory() for t in (q, k, v))
        ho, hl, hc = (torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in (out, lse, cnt))
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        h2d = sum(t.numel() * t.element_size() for t in (hq_, hk_, hv_))
        d2h = sum(t.numel() * t.element_size() for t in (ho, hl, hc))
        n_e2e = max(3, min(args.steps, 30))

        def e2e_step():
            dq.copy_(hq_, non_blocking=True)
            dk.copy_(hk_, non_blocking=True)
            dv.copy_(hv_, non_blocking=True)
            st = fwd(dq, dk, dv, out, lse, cnt)
            if st != 0:
                raise RuntimeError(ssa.status_string(st))
            ho.copy_(out, non_blocking=True)
            hl.copy_(lse, non_blocking=True)
            hc.copy_(cnt, non_blocking=True)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        barrier()
        e0.record(stream)
        for _ in range(n_e2e):
            e2e_step()
        e1.record(stream)
        e1.synchronize()
        barrier()
        ems = reduce_max(e0.elapsed_time(e1), dist, dev)
        e2e = {"value": job_rate(flops_dense, world, ems / n_e2e) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ems / n_e2e,
               "steps": n_e2e}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, lam, args.cpu_budget)

    configs = None
    if world == 1 and not args.no_configs:
        del sets
        torch.cuda.empty_cache()
        with Clocks(local_rank) as clk_sweep:
            configs = sweep_configs(dev, stream)
        configs["_clocks"] = clk_sweep.summary()

    if rank == 0:
        clocks = clk.summary()
        line = {
            "metric": "attn fwd TFLOP/s (dense-equiv)",
            "value": tflops_dense, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": workload_name(w, lam) + (
                           "" if mask_bits is None else
                           f" key blocks by bitmap, {args.exact_blocks} of {nK} per query block" if args.exact_blocks
                           else f" key blocks by bitmap, density {args.mask_density:g}"),
                       "parallelism": f"replicas x{world}",
                       "l2": f"inputs alternate between 2 sets of {set_mb:.0f} MB each (Q, K, V; L2 126 MB)"},
            "executed_tflops": tflops_exec,
            "executed_frac_of_peak": tflops_exec / world / bf16_peak,
            "tiles_skipped_frac": skipped / visited,
            "tiles_visited": visited, "tiles_skipped": skipped,
            "tokens_per_s": tokens,
            "roofline": {"bound": "tensor", "achieved": flops_exec / (ms_step * 1e-3) / 1e12,
                         "peak": bf16_peak, "unit": "TFLOP/s",
                         "frac": flops_exec / (ms_step * 1e-3) / 1e12 / bf16_peak,
                         "traffic": traffic, "peak_source": f"{src} bf16 burst",
                         "kernel": f"ssa::ssa_fwd_kernel<{w.d},{w.Bc},{w.m if w.mode & 2 else 0},0>",
                         "dense_equiv_frac": flops_dense / (ms_step * 1e-3) / 1e12 / bf16_peak,
                         "hbm_frac_of_algorithmic_bytes": None},
            "gpu_launches": args.steps,
            "clocks": clocks,
            "e2e": e2e,
            "cpu_baseline": cpu,
            "kernel_hash": kernel_hash(),
            "configs": configs,
        }
        alg_bytes = 2 * (2 * w.B * w.L * w.Hq * w.d + 2 * w.B * w.L * w.Hkv * w.d) + 4 * w.B * w.Hq * w.L
        line["roofline"]["hbm_frac_of_algorithmic_bytes"] = alg_bytes / (ms_step * 1e-3) / 1e9 / hbm_peak
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
