"""Throughput of the low-bit MoE hot path on B200, one JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

A step is one pass of the whole path over one batch of synthetic tokens. The
default workload is the largest single-GPU layer: the trillion-parameter-shaped
INT4 MoE layer (E=384, top-8, d=7168, f=2048, SwiGLU, T=16384 tokens per GPU):
route -> permute -> fused dequant + grouped GEMM gate/up with SwiGLU -> fused
dequant + grouped GEMM down -> combine. Other workloads (--workload) run the
MXFP4 up-projection, the other token counts, the skewed MXFP4 layer, or
forward + backward with the adapter.

Timing: inputs live in HBM; four independent input sets (weights, tokens,
logits, outputs; together larger than the 126 MB L2) are used in rotation so
no step finds its data in L2. Each step is one CUDA-graph replay; the K timed
steps are bracketed by a barrier and a device synchronize on both sides and
timed with CUDA events on the launching stream; the max over ranks is
reported. With N > 1 GPUs every rank runs its own token batch against the
same (replicated) weights: weak scaling, no collective on the data path.

--impl reference times the CPU oracle (plain float64 numpy) on this machine's host
cores, rank 0 only, on a bounded sample of the same workload.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "grouped low-bit MoE GEMM TFLOP/s and weight GB/s (fraction of roofline)"
ROTATE = 4


def _args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default="trillion_int4_T16384")
    ap.add_argument("--chunk", type=int, default=None)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--prior-art", action="store_true",
                    help="time the temporary-buffer scheme against the fused GEMMs, per chunk size")
    return ap.parse_args()


def _workloads():
    from quantized_rl_fine_b200 import configs as C
    w = {
        "mxfp4_up": C.MXFP4_UP,
        "tiny_int4": C.TINY_INT4,
        "zipf_mxfp4": C.ZIPF_MXFP4,
        "train_int4": C.TRAIN_INT4,
    }
    for T in C.TRILLION_T_SWEEP:
        w[f"trillion_int4_T{T}"] = C.TRILLION_INT4.with_(T=T, name=f"{C.TRILLION_INT4.name}_T{T}")
    # The per-expert shape of the decode step (about 2.7 token rows per active
    # expert) with 48 experts: small enough for a full ncu capture.
    w["trillion_int4_E48_T16"] = C.TRILLION_INT4.with_(
        E=48, T=16, name="trillion_int4_E48_k8_d7168_f2048_T16")
    # The per-expert shape of the T=16384 layer (about 341 token rows per
    # expert) and of the training step (about 85) with 48 experts: the same
    # kernels and tiles, small enough for a full ncu capture.
    w["trillion_int4_E48_T2048"] = C.TRILLION_INT4.with_(
        E=48, T=2048, name="trillion_int4_E48_k8_d7168_f2048_T2048")
    w["train_int4_E48_T512"] = C.TRAIN_INT4.with_(
        E=48, T=512, name="train_int4_adapter_E48_k8_d7168_f2048_T512")
    # Zipf-skewed MXFP4 routing with 64 experts and the same mean of 256 rows
    # per expert as the E=256, T=8192 layer (the ranks' bias is the same, so
    # the head experts hold a larger share of the rows): for a full capture.
    w["zipf_mxfp4_E64_T2048"] = C.ZIPF_MXFP4.with_(
        E=64, T=2048, name="zipf_mxfp4_E64_k8_d4096_f1536_T2048")
    return w


# ----------------------------------------------------------------------------- accounting

def _accounting(cfg, counts):
    """Useful flops and algorithmic bytes of one step from the per-expert row counts."""
    from quantized_rl_fine_b200 import accounting as A
    M = int(sum(counts))
    act = [c for c in counts if c > 0]
    d, f = cfg.d, cfg.f
    if not cfg.swiglu:
        flops = A.gemm_flops(counts, f, d)
        wbytes = A.active_weight_bytes(counts, f, d, cfg.fmt)
        gemm = dict(flops=flops, bytes=wbytes + M * d * 2 + M * f * 2, wbytes=wbytes)
        return dict(flops=flops, wbytes=wbytes, gemm=gemm)
    gu_flops = A.gemm_flops(counts, 2 * f, d)
    dn_flops = A.gemm_flops(counts, d, f)
    gu_w = A.active_weight_bytes(counts, 2 * f, d, cfg.fmt)
    dn_w = A.active_weight_bytes(counts, d, f, cfg.fmt)
    flops = gu_flops + dn_flops + (2 * M * d * 32 if cfg.adapter else 0)
    wbytes = gu_w + dn_w
    if cfg.train:
        flops += gu_flops + dn_flops + (4 * M * d * 32 if cfg.adapter else 0)
        wbytes *= 2
    gemm = dict(flops=gu_flops, bytes=gu_w + M * d * 2 + M * f * 2 + (M * 2 * f * 2 if cfg.train else 0),
                wbytes=gu_w)
    return dict(flops=flops, wbytes=wbytes, gemm=gemm)


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """NVML samples of SM clock and throttle reasons while the timed region runs."""

    REASONS = {
        0x0000000000000004: "sw_power_cap", 0x0000000000000008: "hw_slowdown",
        0x0000000000000020: "sw_thermal_slowdown", 0x0000000000000040: "hw_thermal_slowdown",
        0x0000000000000080: "hw_power_brake_slowdown", 0x0000000000000002: "applications_clocks_setting",
    }

    def __init__(self, cuda_index):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._nv = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(cuda_index)
            want = (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
            for i in range(pynvml.nvmlDeviceGetCount()):
                h = pynvml.nvmlDeviceGetHandleByIndex(i)
                pci = pynvml.nvmlDeviceGetPciInfo(h)
                if (pci.domain, pci.bus, pci.device) == want:
                    self._h = h
                    self._nv = pynvml
                    break
            if self._nv is not None:
                self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nv = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM))
                mask = self._nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if mask & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self._nv is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._nv is not None:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ----------------------------------------------------------------------------- profiles

def _kernel_source_hash():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "quantized_rl_fine_b200", "csrc")
    for name in ("gemm.cu", "dequant.cuh", "common.cuh"):
        with open(os.path.join(csrc, name), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def _profiled_traffic(workload):
    """DRAM bytes per launch of the grouped GEMM from the committed ncu summary,
    when it was taken on the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", f"grouped_qgemm_{workload}.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m_hash = re.search(r"kernel source hash:\s*`?([0-9a-f]{16})", text)
    m_bytes = re.search(r"dram bytes per launch:\s*([0-9.eE+]+)", text)
    if not m_hash or not m_bytes or m_hash.group(1) != _kernel_source_hash():
        return None
    return float(m_bytes.group(1))


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        p = json.load(open(path))
        return dict(hbm=p["hbm_gbs"], tensor=p["bf16_tflops"], tensor_sust=p["bf16_tflops_sustained"],
                    source="measured")
    return dict(hbm=6650.0, tensor=1590.0, tensor_sust=1400.0, source="fallback")


# ----------------------------------------------------------------------------- reference arm

class _HostExperts:
    """Oracle (numpy) view of a weight stack held on the device: one expert is
    copied to the host when the oracle first asks for it."""

    def __init__(self, w):
        self.w, self.fmt, self._cache = w, w.fmt, {}

    def expert(self, e):
        import numpy as np
        import torch
        import oracle as O
        if e not in self._cache:
            packed = self.w.packed[e:e + 1].cpu().numpy()
            sc = self.w.scales[e:e + 1].cpu()
            sc = sc.view(torch.int16).numpy().view(np.uint16) if self.fmt == "int4" else sc.numpy()
            self._cache[e] = O.QWeight(self.fmt, packed, sc)
        return self._cache[e]


def _slice_features(w, e, nf):
    """Expert e of an oracle weight stack, restricted to its first nf rows."""
    import oracle as O
    we = w.expert(e)
    return O.QWeight(we.fmt, we.packed[:, :nf], we.scales[:, :, :nf])


def _oracle_step_sample(cfg, wl_np, n_experts, frac=1.0):
    """One oracle step restricted to the rows of the first n_experts active
    experts; with frac < 1 (one expert), to the first frac of its output
    features as well. Returns (seconds, useful flops of the sample)."""
    import numpy as np
    import oracle as O
    t0 = time.perf_counter()
    topk, gates = O.route_topk(wl_np["logits"], cfg.k)
    g = O.group_by_expert(topk, cfg.E, cfg.chunk_size)
    flops = 0
    for e in g.active[:n_experts]:
        rows = np.arange(g.offsets[e], g.offsets[e + 1])
        xp = wl_np["x"][g.perm_token[rows]]
        re_ = np.zeros(len(rows), dtype=np.int64)
        if not cfg.swiglu:
            nf = max(64, int(cfg.f * frac) // 64 * 64)
            O.grouped_gemm_fwd(xp, re_, _slice_features(wl_np["w_up"], e, nf))
            flops += 2 * len(rows) * nf * cfg.d
            continue
        nf = max(64, int(cfg.f * frac) // 64 * 64)        # H features of the sample
        wgu = wl_np["w_gu"].expert(e)
        gate_up = O.QWeight(wgu.fmt, np.concatenate([wgu.packed[:, :nf],
                                                     wgu.packed[:, cfg.f:cfg.f + nf]], 1),
                            np.concatenate([wgu.scales[:, :, :nf],
                                            wgu.scales[:, :, cfg.f:cfg.f + nf]], 2))
        wd = wl_np["w_d"].expert(e)
        down = O.QWeight(wd.fmt, wd.packed[:, :, :nf // 2], wd.scales[:, :nf // 32, :])
        xa = O.adapter_fwd(xp, re_, wl_np["R"][e:e + 1]) if cfg.adapter else xp
        h, saved = O.grouped_gemm_fwd(xa, re_, gate_up, O.EPI_SWIGLU)
        O.grouped_gemm_fwd(h, re_, down)
        step = 2 * len(rows) * (2 * nf * cfg.d + nf * cfg.d)
        if cfg.train:
            dyp = wl_np["dy"][g.perm_token[rows]]
            dgu = O.grouped_gemm_bwd_dx(dyp, re_, down, O.EPI_SWIGLU_BWD, saved)
            dxa = O.grouped_gemm_bwd_dx(dgu, re_, gate_up)
            if cfg.adapter:
                O.adapter_bwd(xp, dxa, re_, wl_np["R"][e:e + 1], 1)
            step *= 2
        flops += step
    return time.perf_counter() - t0, flops


def _sample_size(cfg, wl, budget_s):
    """(n_experts, frac) whose oracle step takes about budget_s seconds."""
    import oracle as O
    t_one, _ = _oracle_step_sample(cfg, wl, 1)
    topk, _ = O.route_topk(wl["logits"], cfg.k)
    A = O.group_by_expert(topk, cfg.E, cfg.chunk_size).num_active
    if t_one <= budget_s:
        return int(max(1, min(A, budget_s / max(t_one, 1e-4)))), 1.0, A
    return 1, max(64.0 / cfg.f, budget_s / t_one), A


def _numpy_workload(cfg, T, wl=None):
    """The oracle's inputs: the seeded workload (drawn on the GPU when there is
    one, so that the 9.5 GB trillion-shaped base is not drawn on the host),
    with the token tensors on the host and each expert's weights copied to the
    host only when the oracle's sample reaches it."""
    import numpy as np
    import torch
    from quantized_rl_fine_b200 import synth
    if wl is None:
        dev = "cuda" if torch.cuda.is_available() else "cpu"
        wl = synth.make_workload(cfg, dev, T=T)
    out = {"logits": wl["logits"].cpu().numpy(), "x": wl["x"].float().cpu().numpy().astype(np.float64)}
    for key in ("w_up", "w_gu", "w_d"):
        if key in wl:
            out[key] = _HostExperts(wl[key])
    if cfg.adapter:
        out["R"] = wl["adapter"].float().cpu().numpy().astype(np.float64)
    if cfg.train:
        out["dy"] = wl["dy"].float().cpu().numpy().astype(np.float64)
    return out


def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max((i.get("num_threads", 1) for i in threadpool_info()), default=os.cpu_count())
    except Exception:
        return os.cpu_count()


def _cpu_baseline(cfg, budget_s=20.0, wl_dev=None):
    """Oracle throughput on a bounded sample (about budget_s seconds), timed once."""
    wl = _numpy_workload(cfg, cfg.T, wl_dev)
    n, frac, A = _sample_size(cfg, wl, budget_s)
    secs, flops = _oracle_step_sample(cfg, wl, n, frac)
    part = "all of their output features" if frac >= 1.0 else f"{frac:.3f} of its output features"
    return dict(value=flops / secs / 1e12, unit="TFLOP/s", cores=_blas_threads(), kind="oracle",
                sample=f"routing of all {cfg.T} tokens + the rows of {n} of {A} active experts, "
                       f"{part}; one pass of the float64 numpy oracle, "
                       f"{flops / 1e9:.2f} GFLOP in {secs:.2f} s")


def _config_dict(cfg, chunk, world):
    """The workload description both arms print."""
    return {"workload": cfg.name, "E": cfg.E, "k": cfg.k, "d": cfg.d, "f": cfg.f,
            "T_per_gpu": cfg.T, "fmt": cfg.fmt, "chunk_size": chunk,
            "adapter": cfg.adapter, "train": cfg.train,
            "l2": f"{ROTATE} rotating input sets, larger than L2 together",
            "parallelism": f"dp{world} (replicated weights, own tokens per GPU)"}


def run_reference(args, cfg):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    wl = _numpy_workload(cfg, cfg.T)
    per_step = 150.0 / max(1, args.steps + args.warmup)
    n, frac, A = _sample_size(cfg, wl, per_step)
    for _ in range(args.warmup):
        _oracle_step_sample(cfg, wl, n, frac)
    secs = flops = 0.0
    for _ in range(args.steps):
        s, fl = _oracle_step_sample(cfg, wl, n, frac)
        secs += s
        flops += fl
    value = flops / secs / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": secs / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": _config_dict(cfg, args.chunk or cfg.chunk_size, args.gpus),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": _blas_threads(),
                         "kind": "oracle",
                         "sample": f"each step: routing of all {cfg.T} tokens + the GEMMs of "
                                   f"the rows of {n} of {A} active experts"
                                   + ("" if frac >= 1.0 else f", {frac:.3f} of the output features")},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- our arm

def _make_sets(cfg, device, rank):
    from quantized_rl_fine_b200 import synth
    sets = []
    for i in range(ROTATE):
        c = cfg.with_(seed=cfg.seed + 7919 * i + 104729 * rank)
        wl = synth.make_workload(c, device)
        sets.append(wl)
    return sets


def _step_fn(cfg, chunk):
    from quantized_rl_fine_b200 import layer

    def step(wl):
        if not cfg.swiglu:
            return layer.up_projection(wl["x"], wl["logits"], wl["w_up"], cfg.k, chunk)
        st = layer.forward(wl["x"], wl["logits"], wl["w_gu"], wl["w_d"], cfg.k, chunk,
                           adapter=wl.get("adapter"), train=cfg.train)
        if cfg.train:
            bw = layer.backward(st, wl["dy"], wl["w_gu"], wl["w_d"], adapter=wl.get("adapter"))
            st.update(bw)
        return st
    return step


def _launches_per_step(cfg):
    # routing: top-k and the single-pass tail (which also copies the rows) for
    # launches of at most 1024 tokens whose token-by-expert bit matrix fits
    # 8192 words; else top-k, scan, scatter and, without the adapter, the row
    # copy (with the adapter the adapter kernels gather the rows instead).
    words = (cfg.T + 31) // 32
    route = 2 if words <= 32 and words * cfg.E <= 8192 else (3 if cfg.adapter else 4)
    # a forward GEMM runs as two launches (experts of at most 192 rows on the
    # narrow kernel, the rest on the wide one) once the mean expert holds more
    # than 96 rows
    per_gemm = 2 if cfg.T * cfg.k > 96 * cfg.E else 1
    if not cfg.swiglu:
        return route + per_gemm
    n = route + 2 * per_gemm + 1                # gate/up, down, combine
    if cfg.adapter:
        n += 1                                  # adapter apply
    if cfg.train:
        n += 1 + 2 + 1                          # scatter, two bwd GEMMs, unpermute-sum
        if cfg.adapter:
            n += 1                              # adapter backward (dx and dR in one kernel)
    return n


def _check_device(moeq, phase):
    code = moeq.moe_get_device_error()
    if code != 0:
        raise SystemExit(f"device error word {code} after the {phase}: results are not valid")


def run_ours(args, cfg):
    import torch
    import torch.distributed as dist
    from quantized_rl_fine_b200 import moeq
    from quantized_rl_fine_b200.build import build

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    if rank == 0:
        build()
    if world > 1:
        dist.barrier()
    moeq.lib()

    chunk = args.chunk or cfg.chunk_size
    step = _step_fn(cfg, chunk)
    sets = _make_sets(cfg, dev, rank)
    torch.cuda.synchronize()

    # routing statistics of set 0 (outside any timed region)
    r0 = moeq.moe_route_permute(sets[0]["logits"], None, cfg.k, chunk)
    counts = (r0.expert_offsets[1:] - r0.expert_offsets[:-1]).cpu().tolist()
    acc = _accounting(cfg, counts)

    # eager warm-up (sets attributes, builds maps), then one graph per input set
    for wl in sets:
        step(wl)
    torch.cuda.synchronize()
    graphs, keep = [], []
    for wl in sets:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            keep.append(step(wl))
        graphs.append(g)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    # Training with several ranks: the shared adapter's gradient is summed over
    # the ranks after every step (the path's only collective), eagerly after
    # the graph replay so every rank issues the same collectives in order.
    from quantized_rl_fine_b200 import dp as dp_mod
    reduce_grad = cfg.train and cfg.adapter and world > 1

    def run_step(i):
        graphs[i % ROTATE].replay()
        if reduce_grad:
            dp_mod.allreduce_adapter_grad(keep[i % ROTATE]["d_adapter"])

    # Every set's graph runs once before anything reads its outputs (the
    # GEMM-alone and end-to-end phases below replay all sets).
    for i in range(ROTATE):
        run_step(i)
    for i in range(args.warmup):
        run_step(i)
    torch.cuda.synchronize()

    # ---------------------------------------------------------------- timed region
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        t0.record(stream)
        for i in range(args.steps):
            run_step(i)
        t1.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms = t0.elapsed_time(t1)
    if world > 1:
        tt = torch.tensor([ms], device=dev)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        ms = float(tt.item())
    ms_per_step = ms / args.steps
    _check_device(moeq, "timed steps")

    # ---------------------------------------------------------------- dominant kernel alone
    from quantized_rl_fine_b200 import layer
    gemm_graphs = []
    for i, wl in enumerate(sets):
        st = keep[i]
        r = st["routing"]
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            # the layer's own call (its input rows: x_perm, or x through perm_token)
            if not cfg.swiglu:
                moeq.moe_grouped_qgemm_fwd(st["a"], wl["w_up"], r, moeq.EPI_NONE,
                                           a_rows=st["a_rows"])
            else:
                moeq.moe_grouped_qgemm_fwd(st["a"], wl["w_gu"], r, moeq.EPI_SWIGLU,
                                           adapter=wl.get("adapter"), save_gu=cfg.train,
                                           a_rows=st["a_rows"])
        gemm_graphs.append(g)
    for i in range(max(3, args.warmup)):
        gemm_graphs[i % ROTATE].replay()
    torch.cuda.synchronize()
    ka, kb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # About 200 ms of back-to-back launches (at least 20), whatever --steps
    # is, so the kernel's time does not depend on how long the step timing
    # ran and every workload's kernel is timed over the same span.
    ka.record(stream)
    for i in range(10):
        gemm_graphs[i % ROTATE].replay()
    kb.record(stream)
    torch.cuda.synchronize()
    est_ms = ka.elapsed_time(kb) / 10
    n_k = max(20, int(200.0 / max(est_ms, 1e-3)) + 1)
    ka.record(stream)
    for i in range(n_k):
        gemm_graphs[i % ROTATE].replay()
    kb.record(stream)
    torch.cuda.synchronize()
    k_ms = ka.elapsed_time(kb) / n_k
    _check_device(moeq, "grouped GEMM alone")

    # ---------------------------------------------------------------- end to end via host buffers
    host = []
    for wl in sets:
        hx = wl["x"].cpu().pin_memory()
        hl = wl["logits"].cpu().pin_memory()
        hy = wl["dy"].cpu().pin_memory() if cfg.train else None
        host.append((hx, hl, hy))
    out_key = "out" if not cfg.swiglu else ("dx" if cfg.train else "y")
    out_shape = keep[0][out_key].shape
    hout = [torch.empty(out_shape, dtype=torch.bfloat16).pin_memory() for _ in range(ROTATE)]
    h2d = sum(t.numel() * t.element_size() for t in host[0] if t is not None)
    d2h = hout[0].numel() * hout[0].element_size()

    # Three streams, as an input pipeline runs them: the host->device copy of
    # a step's inputs, the step itself and the device->host read of its result
    # overlap with those of neighbouring steps. Each input set's buffers are
    # reused only after its previous step and read-back have finished.
    s_in = torch.cuda.Stream(device=dev)
    s_out = torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(ROTATE)]
    ev_done = [torch.cuda.Event() for _ in range(ROTATE)]
    ev_out = [torch.cuda.Event() for _ in range(ROTATE)]
    used = [False] * ROTATE

    def e2e_step(i):
        j = i % ROTATE
        hx, hl, hy = host[j]
        wl = sets[j]
        if used[j]:
            s_in.wait_event(ev_done[j])
        with torch.cuda.stream(s_in):
            wl["x"].copy_(hx, non_blocking=True)
            wl["logits"].copy_(hl, non_blocking=True)
            if hy is not None:
                wl["dy"].copy_(hy, non_blocking=True)
            ev_in[j].record(s_in)
        stream.wait_event(ev_in[j])
        if used[j]:
            stream.wait_event(ev_out[j])
        run_step(i)
        ev_done[j].record(stream)
        s_out.wait_event(ev_done[j])
        with torch.cuda.stream(s_out):
            hout[j].copy_(keep[j][out_key], non_blocking=True)
            ev_out[j].record(s_out)
        used[j] = True

    def e2e_drain():
        for j in range(ROTATE):
            if used[j]:
                stream.wait_event(ev_out[j])

    for i in range(max(3, args.warmup)):
        e2e_step(i)
    e2e_drain()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_in.wait_event(e0)                      # no copy starts before the timed region
    for i in range(args.steps):
        e2e_step(i)
    e2e_drain()                              # every read-back is inside the timed region
    e1.record(stream)
    torch.cuda.synchronize()
    e_ms = e0.elapsed_time(e1)
    if world > 1:
        tt = torch.tensor([e_ms], device=dev)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        e_ms = float(tt.item())
    _check_device(moeq, "end-to-end steps")

    # ---------------------------------------------------------------- report
    del graphs, gemm_graphs
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    peaks = _peaks()
    step_flops = acc["flops"]
    value = world * step_flops / (ms_per_step * 1e-3) / 1e12
    gemm = acc["gemm"]
    k_bytes_rate = gemm["bytes"] / (k_ms * 1e-3) / 1e9
    k_flop_rate = gemm["flops"] / (k_ms * 1e-3) / 1e12
    t_hbm = gemm["bytes"] / (peaks["hbm"] * 1e9)
    t_tc = gemm["flops"] / (peaks["tensor"] * 1e12)
    if t_hbm >= t_tc:
        roof = {"bound": "hbm", "achieved": k_bytes_rate, "peak": peaks["hbm"], "unit": "GB/s"}
    else:
        roof = {"bound": "tensor", "achieved": k_flop_rate, "peak": peaks["tensor"], "unit": "TFLOP/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = _profiled_traffic(args.workload)
    roof["kernel"] = "grouped_qgemm_kernel (fwd" + (", SwiGLU" if cfg.swiglu else "") + ")"
    roof["kernel_ms"] = k_ms
    roof["kernel_launches_timed"] = n_k
    roof["algorithmic_bytes"] = gemm["bytes"]
    roof["algorithmic_flops"] = gemm["flops"]
    roof["peak_source"] = peaks["source"] + " (burst)"
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": _config_dict(cfg, chunk, world),
        "weight_gbs": world * acc["wbytes"] / (ms_per_step * 1e-3) / 1e9,
        "roofline": roof,
        "e2e": {"value": world * step_flops / (e_ms / args.steps * 1e-3) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e_ms / args.steps,
                "pipelining": "input copy, step and read-back of neighbouring steps overlap "
                              "on three streams"},
        "gpu_launches": _launches_per_step(cfg) * args.steps,
        "clocks": clocks.summary(),
    }
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = _cpu_baseline(cfg, wl_dev=sets[0])
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- prior-art comparator

def run_prior_art(args, cfg):
    """One JSON line per chunk size C: the Orbit article's temporary-buffer
    scheme (chunk of C experts dequantized to BF16, cuBLAS GEMMs, buffer
    released) against this library's fused GEMMs on the same routed rows, with
    the temporary memory each needs. Eager launches, CUDA events, median of
    the repetitions; the weights (GBs) are far larger than L2."""
    import torch
    from quantized_rl_fine_b200 import moeq, prior_art, synth
    from quantized_rl_fine_b200.build import build
    build()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    wl = synth.make_workload(cfg, dev)
    w_first = wl["w_gu"] if cfg.swiglu else wl["w_up"]
    reps = max(3, min(args.steps, 10))

    def timed(fn):
        ts = []
        for _ in range(reps + 1):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        return statistics.median(ts[1:])

    for C in (8, 16, 32):
        r = moeq.moe_route_permute(wl["logits"], wl["x"], cfg.k, C)
        M = r.x_perm.shape[0]
        h = torch.empty((M, cfg.f), dtype=torch.bfloat16, device=dev)
        y = torch.empty((M, cfg.d if cfg.swiglu else cfg.f), dtype=torch.bfloat16, device=dev)

        def fused():   # the layer's calls (no adapter: the permuted rows)
            if cfg.swiglu:
                moeq.moe_grouped_qgemm_fwd(r.x_perm, w_first, r, moeq.EPI_SWIGLU, out=h)
                moeq.moe_grouped_qgemm_fwd(h, wl["w_d"], r, moeq.EPI_NONE, out=y)
            else:
                moeq.moe_grouped_qgemm_fwd(r.x_perm, w_first, r, moeq.EPI_NONE, out=y)
        got = {}

        def prior():
            got["y"], got["peak"] = prior_art.forward(r.x_perm, r, w_first, wl.get("w_d"), C,
                                                      swiglu=cfg.swiglu)
        t_fused = timed(fused)
        t_prior = timed(prior)
        diff = (got["y"].float() - y.float()).abs().max().item()
        print(json.dumps({
            "comparator": "temporary BF16 buffer per chunk of active experts + cuBLAS GEMMs",
            "workload": cfg.name, "chunk_size": C, "reps": reps,
            "prior_art_ms": t_prior, "fused_ms": t_fused, "fused_speedup": t_prior / t_fused,
            "prior_art_peak_temp_bytes": got["peak"], "fused_temp_bytes": 0,
            "max_abs_diff_of_per_slot_outputs": diff}), flush=True)
        del got


def main():
    args = _args()
    cfg = _workloads()[args.workload]
    if args.prior_art:
        run_prior_art(args, cfg)
        return
    if args.impl == "reference":
        run_reference(args, cfg)
    else:
        run_ours(args, cfg)


if __name__ == "__main__":
    main()
