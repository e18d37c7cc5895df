"""Benchmark of the JEPA ViT encoder forward on B200.

One step = one forward of one batch of the workload through jepa_b200_encode
(patch-embed, all blocks, final norm, pooling), inputs resident in HBM.
Default workload: LeVJEPA ViT-L/16, 16 frames 224^2 (3137 tokens with the CLS
sink), block-causal mask, f16 weights, batch 4, CLS output.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

Prints one JSON line (rank 0).  Multi-GPU runs are replicas (one process per
GPU via torchrun; each GPU encodes its own batch; no data-path collective).
The reference arm times the float64 CPU oracle on the host cores on a bounded
sample of the same workload.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import glob
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from jepa_video_encoder_b200 import synth  # noqa: E402

METRIC = "ViT-L/16 encoder tokens/s & clips/s on 1 B200; % of dense f16/bf16 TC peak"
DEFAULT_WORKLOAD = synth.LEVJEPA_VIT_L.name
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
NOMINAL_DENSE_F16_TFLOPS = 2250.0   # B200 dense f16 / bf16 tensor rate as specified (no sparsity)


def max_over_ranks(value: float, world: int, device=None) -> float:
    """The largest of every rank's value (all-reduce MAX over the process
    group); a timed region lasts as long as its slowest rank."""
    if world <= 1:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank_step: int, world: int, steps: int, total_ms: float) -> float:
    """Units all replicas processed per second: every rank encodes its own
    batch each step (weak scaling), the time is the slowest rank's."""
    return world * units_per_rank_step * steps / (total_ms / 1000.0)


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def peak_dense_of(peaks) -> float:
    return float(peaks.get("bf16_tflops"))


def _flops(cfg) -> dict:
    """Algorithmic FLOPs per clip by kernel class (attention counts only the
    allowed query/key pairs of the mask)."""
    import numpy as np
    N, D, M, L = cfg.n_tokens, cfg.dim, cfg.mlp, cfg.depth
    if cfg.mask == "block_causal":
        pf, c = cfg.patches_per_slot, (1 if cfg.has_cls else 0)
        slots = np.arange(cfg.n_patches) // pf
        pairs = int(((slots + 1) * pf).sum()) + (N if c else 0)
    else:
        pairs = N * N
    f = {
        "patch_embed": 2.0 * cfg.n_patches * cfg.patch_k * D,
        "gemm_qkv": 2.0 * N * D * 3 * D * L,
        "attention": 4.0 * pairs * D * L,
        "gemm_out": 2.0 * N * D * D * L,
        "gemm_up": 2.0 * N * D * M * L,
        "gemm_down": 2.0 * N * M * D * L,
    }
    if cfg.has_head:
        f["head"] = cfg.head_sa_blocks * (24.0 * N * D * D + 4.0 * N * N * D) + 4.0 * N * D * D
    return f


_CLOCK_FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                 "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                 "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


def _clock_sampler_start(path):
    try:
        f = open(path, "w")
        return subprocess.Popen(["nvidia-smi", f"--query-gpu={_CLOCK_FIELDS}", "--format=csv,noheader,nounits",
                                 "-lms", "50"], stdout=f, stderr=subprocess.DEVNULL), f
    except Exception:
        return None, None


def parse_clock_log(path, gpu_index, t0=None, t1=None):
    """Median SM clock, max clock and the throttle reasons seen in an nvidia-smi
    log of _CLOCK_FIELDS.  With t0 / t1 (host epoch seconds) only the samples
    taken inside [t0, t1] count; if none falls inside, all of them do and
    ``in_region`` says so."""
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    rows = []
    for line in open(path):
        parts = [q.strip() for q in line.split(",")]
        if len(parts) < 10 or parts[1] != str(gpu_index):
            continue
        try:
            sm, mx = float(parts[2]), float(parts[3])
        except ValueError:
            continue
        ts = None  # a sample whose time cannot be read still counts in the fallback
        for fmt in ("%Y/%m/%d %H:%M:%S.%f", "%Y/%m/%d %H:%M:%S"):
            try:
                ts = datetime.datetime.strptime(parts[0], fmt).timestamp()
                break
            except ValueError:
                pass
        rows.append((ts, sm, mx, [n for n, v in zip(names, parts[6:10]) if v.lower() == "active"]))
    if not rows:
        return None
    inside = [r for r in rows if t0 is not None and t1 is not None and r[0] is not None and t0 <= r[0] <= t1]
    use = inside or rows
    return {"sm_mhz": statistics.median(r[1] for r in use), "sm_max_mhz": max(r[2] for r in use),
            "reasons": sorted({n for r in use for n in r[3]}), "samples": len(use),
            "in_region": bool(inside)}


def _clock_sampler_stop(proc, fh, path, gpu_index, t0=None, t1=None):
    if proc is None:
        return None
    proc.terminate()
    try:
        proc.wait(timeout=5)
    except Exception:
        proc.kill()
    fh.close()
    return parse_clock_log(path, gpu_index, t0, t1)


# The sources each kernel class is compiled from: a traffic figure stays valid
# while these files are unchanged.
_CLASS_SOURCES = {
    "attention": ("attention.cu", "common.cuh", "internal.h"),
    "layernorm": ("norm_pool.cu", "common.cuh", "internal.h"),
    "pool_head": ("head.cu", "norm_pool.cu", "common.cuh", "internal.h"),
}
_GEMM_SOURCES = ("gemm.cu", "common.cuh", "internal.h")


_C_TOKENS = re.compile(r'//[^\n]*|/\*.*?\*/|"(?:\\.|[^"\\\n])*"|\'(?:\\.|[^\'\\\n])*\'', re.S)


def code_text(src: str) -> str:
    """C / C++ / CUDA source without its comments, each line stripped of
    leading and trailing blanks, blank lines dropped: what a comment edit
    leaves unchanged.  String and character literals are kept as they are."""
    out = _C_TOKENS.sub(lambda m: " " if m.group(0)[0] == "/" else m.group(0), src)
    return "\n".join(ln.strip() for ln in out.splitlines() if ln.strip())


def hash_sources(texts) -> str:
    h = hashlib.sha256()
    for t in texts:
        h.update(code_text(t).encode())
        h.update(b"\0")
    return h.hexdigest()[:16]


def _src_hash(kernel_class=None):
    names = _CLASS_SOURCES.get(kernel_class, _GEMM_SOURCES if kernel_class and (
        kernel_class.startswith("gemm_") or kernel_class == "patch_embed") else None)
    csrc = os.path.join(ROOT, "jepa_video_encoder_b200", "csrc")
    paths = [os.path.join(csrc, n) for n in names] if names else sorted(glob.glob(os.path.join(csrc, "*")))
    paths.append(os.path.join(ROOT, "include", "jepa_b200.h"))
    texts = []
    for path in paths:
        with open(path, encoding="utf-8") as f:
            texts.append(f.read())
    return hash_sources(texts)


def _traffic(kernel_class, cfg_name):
    """DRAM bytes per launch of a kernel class from the committed ncu summary
    (profiles/traffic.txt), valid only for the kernel sources it was taken on."""
    p = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(p):
        return None
    src = _src_hash(kernel_class)
    for line in open(p):
        parts = line.split()
        if len(parts) >= 4 and not line.startswith("#") and parts[0] == kernel_class and parts[1] == cfg_name \
                and parts[2] == src:
            return float(parts[3])
    return None


def _oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] + [os.cpu_count() or 1])
    except Exception:
        return os.cpu_count() or 1


def _load_avg():
    try:
        return os.getloadavg()[0]
    except OSError:
        return None


def cpu_oracle_clip(cfg, table=None):
    """Time the float64 oracle on one whole clip of the workload: patch-embed,
    every block, final norm (the workload's full forward for one clip; the
    clip is the bounded sample, the batch being B such clips).  ``table`` (a
    table_dict of the workload) saves regenerating the inputs; making the
    inputs and decoding the weights are not timed."""
    import numpy as np
    from oracle import jepa_oracle as orc
    if table is None:
        table = synth.table_dict(synth.make_tensor_table(cfg))
    pix = synth.make_pixels(cfg, batch=1).astype(np.float64)
    W = {n: orc.tensor_f64(t) for n, t in table.items() if not n.startswith("head.")}
    t0 = time.perf_counter()
    orc.encoder(cfg, W, pix)
    t_clip = time.perf_counter() - t0
    return {"value": cfg.n_tokens / t_clip, "unit": "tokens/s", "cores": _oracle_threads(), "kind": "oracle",
            "clips_per_s": 1.0 / t_clip, "host_cpus": os.cpu_count(), "load_avg_1m": _load_avg(),
            "sample": f"1 clip of the batch: patch-embed, all {cfg.depth} blocks and the final norm in float64 "
                      f"numpy, timed whole ({t_clip:.1f} s)"}


def cpu_oracle_block_step(cfg, W, x, blk, allow, rope_pos):
    """One step of the reference arm: block ``blk`` of one clip in the
    float64 oracle; returns (output, seconds)."""
    from oracle import jepa_oracle as orc
    t0 = time.perf_counter()
    y = orc.block(x, W, f"enc.blk.{blk}.", cfg.heads, cfg.ln_eps, allow, rope_pos)
    return y, time.perf_counter() - t0


def run_config(cfg, world: int, l2: str) -> dict:
    """The workload a line measures; both arms report the same keys."""
    return {"workload": cfg.name, "batch_per_gpu": cfg.batch, "global_batch": cfg.batch * world,
            "tokens_per_clip": cfg.n_tokens, "weights": cfg.weights,
            "activations": "bf16" if cfg.act_bf16 else "f16", "mask": cfg.mask, "pool": cfg.pool,
            "parallelism": f"replicas x{world}", "l2": l2}


def run_reference(args, cfg, rank, world):
    """The oracle on the host cores.  A step is one block of one clip (blocks
    taken in order, wrapping at the depth), so K steps stay a bounded run; the
    rate is one clip's tokens over the time of its whole forward built from
    the measured parts: patch-embed + final norm (timed once) + depth x the
    mean block step."""
    if rank != 0:
        return 0
    import numpy as np
    from oracle import jepa_oracle as orc
    table = synth.table_dict(synth.make_tensor_table(cfg))   # the inputs, generated once
    W = {n: orc.tensor_f64(t) for n, t in table.items() if not n.startswith("head.")}
    pix = synth.make_pixels(cfg, batch=1).astype(np.float64)
    allow = orc.encoder_allow(cfg)
    rope_pos = orc.rope_positions(cfg) if cfg.rope else None
    t0 = time.perf_counter()
    x = orc.embed(cfg, W, pix)
    t_embed = time.perf_counter() - t0
    t0 = time.perf_counter()
    orc.layer_norm(x, W["enc.norm.weight"], W["enc.norm.bias"], cfg.ln_eps)
    t_norm = time.perf_counter() - t0
    blk = 0
    for _ in range(max(0, args.warmup)):
        x, _t = cpu_oracle_block_step(cfg, W, x, blk % cfg.depth, allow, rope_pos)
        blk += 1
    step_s = []
    for _ in range(max(1, args.steps)):
        x, t = cpu_oracle_block_step(cfg, W, x, blk % cfg.depth, allow, rope_pos)
        step_s.append(t)
        blk += 1
    t_block = statistics.mean(step_s)
    t_clip = t_embed + t_norm + cfg.depth * t_block
    v = cfg.n_tokens / t_clip
    sample = (f"1 clip, one of its {cfg.depth} blocks per step in float64 numpy; rate = tokens of the clip / "
              f"(patch-embed {t_embed:.2f} s + final norm {t_norm:.2f} s + {cfg.depth} x mean step "
              f"{t_block:.2f} s)")
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * t_block,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": run_config(cfg, world, l2="not applicable (host CPU run)"),
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": _oracle_threads(), "kind": "oracle",
                             "sample": sample, "host_cpus": os.cpu_count(), "load_avg_1m": _load_avg()},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args, cfg, rank, world, local_rank):
    import numpy as np
    import torch
    import jepa_video_encoder_b200 as jb
    from jepa_video_encoder_b200 import build as jbuild

    if rank == 0 and not os.path.exists(jbuild.LIB):
        jbuild.build()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    table = synth.make_tensor_table(cfg)
    pix_np = synth.make_pixels(cfg)
    model = jb.Model(cfg, table, device=local_rank, quant_f16_copy=args.quant_f16_copy)
    pixels = torch.from_numpy(pix_np).to(dev)
    out = torch.empty(model.out_shape(cfg.batch, cfg.pool), dtype=torch.float32, device=dev)
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=dev)   # 256 MiB > L2
    stream = torch.cuda.current_stream(dev)

    def step():
        model.encode(pixels, pool=cfg.pool, out=out, stream=stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(dev)
    if model.sync_status(stream) != 0:
        raise RuntimeError("device error during warm-up")
    if args.forward_only:   # a fixed number of plain forwards, for profiler launch lists
        for _ in range(args.steps):
            step()
        torch.cuda.synchronize(dev)
        st = model.sync_status(stream)
        model.close()
        return 0 if st == 0 else 1

    # ---- timed region: K steps, each between CUDA events, L2 flushed between steps
    clock_path = (args.clock_log.replace("{rank}", str(rank)) if args.clock_log else
                  os.path.join(tempfile.gettempdir(), f"jepa_clocks_rank{rank}.csv"))
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    proc, fh = _clock_sampler_start(clock_path)
    time.sleep(0.3)
    launches = 0
    t_region0 = time.time()
    for k in range(args.steps):
        flush.zero_()
        ev[k][0].record(stream)
        step()
        ev[k][1].record(stream)
        launches += model.last_launch_count()
    torch.cuda.synchronize(dev)
    t_region1 = time.time()
    clocks = _clock_sampler_stop(proc, fh, clock_path, local_rank, t_region0, t_region1)
    if world > 1:
        torch.distributed.barrier()
    if model.sync_status(stream) != 0:
        raise RuntimeError("device error in the timed region")
    ms_steps = [a.elapsed_time(b) for a, b in ev]
    total_ms = max_over_ranks(sum(ms_steps), world, dev)
    ms_per_step = total_ms / args.steps
    value = whole_job_rate(cfg.batch * cfg.n_tokens, world, args.steps, total_ms)

    # ---- per-kernel timing pass (event pairs around every launch)
    model.set_profiling(True)
    prof = {k: [0.0, 0] for k in jb._abi.KERNEL_CLASSES}
    for k in range(args.steps):
        flush.zero_()
        step()
        for kc, (ms, n) in model.profile_read().items():
            prof[kc][0] += ms
            prof[kc][1] += n
    model.set_profiling(False)

    # ---- end to end through the public API from pinned host memory
    pix_host = torch.from_numpy(pix_np).pin_memory()
    out_host = torch.empty(tuple(out.shape), dtype=torch.float32).pin_memory()
    for _ in range(2):
        model.encode_host(pix_host, pool=cfg.pool, out=out_host, stream=stream)
    e2e_ms = []
    for _ in range(args.steps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        model.encode_host(pix_host, pool=cfg.pool, out=out_host, stream=stream)
        b.record(stream)
        b.synchronize()
        e2e_ms.append(a.elapsed_time(b))
    e2e_value = whole_job_rate(cfg.batch * cfg.n_tokens, world, args.steps, max_over_ranks(sum(e2e_ms), world, dev))

    if rank != 0:
        model.close()
        return 0

    peaks, peak_src = _peaks()
    fl = _flops(cfg)
    B = cfg.batch
    total_flop = B * sum(fl.values())
    tflops = total_flop / (ms_per_step / 1000.0) / 1e12
    # dominant kernel class by measured time
    per_class = {k: v for k, v in prof.items() if v[1] > 0}
    dom = max(per_class, key=lambda k: per_class[k][0])
    dom_ms, dom_n = per_class[dom]
    avg_ms = dom_ms / dom_n
    if dom in fl:
        per_launch = B * fl[dom] / (cfg.depth if dom.startswith("gemm") or dom == "attention" else 1)
        achieved = per_launch / (avg_ms / 1000.0) / 1e12
        # the burst figure: this step is short (well under a second) and runs
        # near the maximum clock; the sustained figure (seconds under the
        # power cap) is reported beside it
        peak = float(peaks.get("bf16_tflops"))
        peak_sus = float(peaks.get("bf16_tflops_sustained", peak))
        roof = {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": _traffic(dom, cfg.name),
                "flop_per_launch": per_launch, "avg_launch_ms": avg_ms,
                "peak_source": f"{peak_src} bf16 burst",
                "peak_sustained": peak_sus, "frac_sustained": achieved / peak_sus}
    else:
        roof = {"bound": "hbm", "kernel": dom, "achieved": None, "peak": float(peaks["hbm_gbs"]), "unit": "GB/s",
                "frac": None, "traffic": None}
    kernels = {k: {"ms_per_step": v[0] / args.steps, "launches_per_step": v[1] / args.steps}
               for k, v in per_class.items()}
    for k in kernels:
        if k in fl and kernels[k]["ms_per_step"] > 0:
            kernels[k]["tflops"] = B * fl[k] / (kernels[k]["ms_per_step"] / 1000.0) / 1e12

    # attention + GEMMs together: their algorithmic FLOPs over their summed
    # event-timed launch durations
    tc_classes = [k for k in per_class if k == "attention" or k.startswith("gemm_")]
    tc_ms = sum(per_class[k][0] for k in tc_classes) / args.steps
    tc_flop = B * sum(fl[k] for k in tc_classes if k in fl)
    attn_gemm = None
    if tc_ms > 0:
        tc_tf = tc_flop / (tc_ms / 1000.0) / 1e12
        attn_gemm = {"tflops": tc_tf, "frac": tc_tf / peak_dense_of(peaks),
                     "frac_sustained": tc_tf / float(peaks.get("bf16_tflops_sustained", peak_dense_of(peaks))),
                     "ms_per_step": tc_ms, "classes": tc_classes}

    cpu = cpu_oracle_clip(cfg) if (world == 1 and not args.no_cpu) else None
    peak_dense = float(peaks.get("bf16_tflops"))
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": ms_per_step,
        "ms_per_step_min": min(ms_steps), "ms_per_step_sd": statistics.pstdev(ms_steps),
        "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if cfg.act_bf16 else "f16", "data": "synthetic",
        "config": dict(run_config(cfg, world, l2="flushed between steps (256 MiB write)"),
                       **({"quant_f16_copy": bool(args.quant_f16_copy)} if cfg.weights in ("q8_0", "q4_0") else {})),
        "weight_bytes": model.n_bytes,
        "clips_per_s": world * B * args.steps / (total_ms / 1000.0),
        "tflops": tflops, "tc_peak_frac": tflops / peak_dense,
        "tc_peak": {"value": peak_dense, "source": f"{peak_src} bf16 burst"},
        "tc_peak_frac_nominal": tflops / NOMINAL_DENSE_F16_TFLOPS,
        "roofline": roof,
        "attn_gemm": attn_gemm,
        "kernels": kernels,
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": "tokens/s",
                "h2d_bytes_per_step": int(pix_host.numel() * 4), "d2h_bytes_per_step": int(out_host.numel() * 4)},
        "gpu_launches": launches,
        "clocks": clocks,
        "when": datetime.datetime.now(datetime.timezone.utc).strftime("%Y-%m-%dT%H:%M:%S.%fZ"),
    }
    print(json.dumps(line), flush=True)
    model.close()
    return 0


def _pred_flops(pc) -> dict:
    """Algorithmic FLOPs per clip of the masked predictor by kernel class
    (attention at the predictor's head dim, every (query, key) pair)."""
    nc, nt = len(pc.ctx_idx), len(pc.tgt_idx)
    L, D, M, De, d = nc + nt, pc.dim, pc.mlp, pc.enc.dim, pc.depth
    return {"patch_embed": 2.0 * nc * De * D, "gemm_qkv": 2.0 * L * D * 3 * D * d, "attention": 4.0 * L * L * D * d,
            "gemm_out": 2.0 * L * D * D * d, "gemm_up": 2.0 * L * D * M * d, "gemm_down": 2.0 * L * M * D * d,
            "pool_head": 2.0 * nt * D * De}


def run_predictor(args, pc, rank, world, local_rank):
    """The masked predictor alone on seeded encoder-output tokens resident in
    HBM: one step = one jepa_b200_predict of the batch; the rate counts the
    predicted target tokens."""
    import torch
    import numpy as np
    import jepa_video_encoder_b200 as jb
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    table = synth.make_tensor_table(pc.enc) + synth.make_predictor_table(pc)
    model = jb.Model(pc.enc, table, device=local_rank, predictor=pc)
    tok_np = synth.make_predictor_tokens(pc)
    tokens = torch.from_numpy(tok_np).to(dev)
    ci, ti = pc.ctx_idx, pc.tgt_idx
    out = torch.empty((pc.batch, len(ti), pc.enc.dim), dtype=torch.float32, device=dev)
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    for _ in range(max(3, args.warmup)):
        model.predict(tokens, ci, ti, out=out, stream=stream)
    torch.cuda.synchronize(dev)
    if model.sync_status(stream) != 0:
        raise RuntimeError("device error during warm-up")
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    clock_path = os.path.join(tempfile.gettempdir(), f"jepa_clocks_rank{rank}.csv")
    proc, fh = _clock_sampler_start(clock_path)
    time.sleep(0.3)
    launches = 0
    t0 = time.time()
    for k in range(args.steps):
        flush.zero_()
        ev[k][0].record(stream)
        model.predict(tokens, ci, ti, out=out, stream=stream)
        ev[k][1].record(stream)
        launches += model.last_launch_count()
    torch.cuda.synchronize(dev)
    clocks = _clock_sampler_stop(proc, fh, clock_path, local_rank, t0, time.time())
    if model.sync_status(stream) != 0:
        raise RuntimeError("device error in the timed region")
    ms_steps = [a.elapsed_time(b) for a, b in ev]
    total_ms = max_over_ranks(sum(ms_steps), world, dev)
    units = pc.batch * len(ti)
    value = whole_job_rate(units, world, args.steps, total_ms)
    model.set_profiling(True)
    prof = {k: [0.0, 0] for k in jb._abi.KERNEL_CLASSES}
    for k in range(args.steps):
        flush.zero_()
        model.predict(tokens, ci, ti, out=out, stream=stream)
        for kc, (ms, n) in model.profile_read().items():
            prof[kc][0] += ms
            prof[kc][1] += n
    model.set_profiling(False)
    if rank != 0:
        model.close()
        return 0
    peaks, peak_src = _peaks()
    fl = _pred_flops(pc)
    B = pc.batch
    kernels = {k: {"ms_per_step": v[0] / args.steps, "launches_per_step": v[1] / args.steps}
               for k, v in prof.items() if v[1] > 0}
    for k in kernels:
        if k in fl and kernels[k]["ms_per_step"] > 0:
            kernels[k]["tflops"] = B * fl[k] / (kernels[k]["ms_per_step"] / 1000.0) / 1e12
    ms_per_step = total_ms / args.steps
    tflops = B * sum(fl.values()) / (ms_per_step / 1000.0) / 1e12
    cpu = None
    if world == 1 and not args.no_cpu:
        from oracle import jepa_oracle as orc
        W = orc.weights_f64([t for t in table if t.name.startswith("pred.")])
        tc = time.perf_counter()
        orc.predictor(pc, W, tok_np[:1].astype(np.float64), ci, ti)
        t_clip = time.perf_counter() - tc
        cpu = {"value": len(ti) / t_clip, "unit": "target tokens/s", "cores": _oracle_threads(), "kind": "oracle",
               "sample": f"1 clip: the whole predictor in float64 numpy, timed whole ({t_clip:.1f} s)"}
    line = {"metric": "masked-predictor target tokens/s on 1 B200", "value": value, "unit": "target tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms_per_step,
            "ms_per_step_min": min(ms_steps), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f16", "data": "synthetic",
            "config": {"workload": pc.name, "batch_per_gpu": B, "n_ctx": len(ci), "n_tgt": len(ti),
                       "pred_dim": pc.dim, "pred_depth": pc.depth, "pred_heads": pc.heads, "weights": pc.weights,
                       "l2": "flushed between steps (256 MiB write)"},
            "tflops": tflops, "tc_peak_frac": tflops / peak_dense_of(peaks), "kernels": kernels,
            "cpu_baseline": cpu, "gpu_launches": launches, "clocks": clocks,
            "when": datetime.datetime.now(datetime.timezone.utc).strftime("%Y-%m-%dT%H:%M:%S.%fZ")}
    print(json.dumps(line), flush=True)
    model.close()
    return 0


def _wm_flops_per_call(wc, T: int) -> float:
    """Algorithmic FLOPs of one LeWM predictor call over T frames of one
    candidate (matrix products, the causal attention's T (T + 1) / 2 pairs)."""
    D, M, H = wc.dim, wc.mlp, wc.pred_hidden
    per_row_block = 2.0 * (6 * D * D + 3 * D * D + D * D + 2 * D * M)
    attn = 4.0 * D * T * (T + 1) / 2 * wc.depth
    return T * (wc.depth * per_row_block + 2.0 * D * D + 2.0 * wc.action_dim * D + 4.0 * D * H) + attn


def _wm_tile_bytes(wc) -> int:
    """Weight bytes one CTA streams per predictor call: every 128-row x
    64-column f16 tile the fused kernel loads (adaLN chunks start on tile
    boundaries, so a 192-wide chunk takes two tiles)."""
    D, M, H = wc.dim, wc.mlp, wc.pred_hidden
    tc = -(-D // 128)
    kd = D // 64
    t = tc * kd + wc.depth * (6 * tc * kd + -(-3 * D // 128) * kd + tc * kd + -(-M // 128) * kd + tc * (M // 64))
    t += -(-H // 128) * kd + tc * (H // 64)
    return t * 16384


def run_world_model(args, wc, rank, world, local_rank):
    """The LeWM world model alone on seeded states and actions resident in
    HBM: one step = one jepa_b200_lewm_predict (wc.steps == 0) or one whole
    jepa_b200_lewm_rollout of every candidate, each a single kernel launch;
    the rate counts predictor calls (one pass over a candidate's window)."""
    import torch
    import jepa_video_encoder_b200 as jb
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    table = synth.make_tensor_table(wc.enc) + synth.make_world_model_table(wc)
    model = jb.Model(wc.enc, table, device=local_rank, world_model=wc)
    st_np, ac_np = synth.make_world_model_inputs(wc)
    st, ac = torch.from_numpy(st_np).to(dev), torch.from_numpy(ac_np).to(dev)
    C = wc.candidates
    calls = C * (wc.steps if wc.steps > 0 else 1)
    out = torch.empty((C, wc.steps if wc.steps > 0 else wc.frames, wc.dim), dtype=torch.float32, device=dev)
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        if wc.steps > 0:
            model.lewm_rollout(st, ac, wc.steps, out=out, stream=stream)
        else:
            model.lewm_predict(st, ac, out=out, stream=stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(dev)
    if model.sync_status(stream) != 0:
        raise RuntimeError("device error during warm-up")
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    torch.cuda.synchronize(dev)
    clock_path = os.path.join(tempfile.gettempdir(), f"jepa_clocks_rank{rank}.csv")
    proc, fh = _clock_sampler_start(clock_path)
    time.sleep(0.3)
    launches = 0
    t0 = time.time()
    for k in range(args.steps):
        flush.zero_()
        ev[k][0].record(stream)
        step()
        ev[k][1].record(stream)
        launches += model.last_launch_count()
    torch.cuda.synchronize(dev)
    clocks = _clock_sampler_stop(proc, fh, clock_path, local_rank, t0, time.time())
    if model.sync_status(stream) != 0:
        raise RuntimeError("device error in the timed region")
    ms_steps = [a.elapsed_time(b) for a, b in ev]
    total_ms = max_over_ranks(sum(ms_steps), world, dev)
    value = whole_job_rate(calls, world, args.steps, total_ms)
    if rank != 0:
        model.close()
        return 0
    ms_per_step = total_ms / args.steps
    # FLOPs: the window grows from `frames` (capped at the window) during a rollout
    if wc.steps > 0:
        fl = sum(_wm_flops_per_call(wc, min(wc.window, wc.frames + s)) for s in range(wc.steps)) * C
    else:
        fl = _wm_flops_per_call(wc, wc.frames) * C
    cpc = 32 // (min(wc.window, wc.frames + wc.steps - 1) if wc.steps > 0 else wc.frames)
    ctas = -(-C // cpc)
    tile_bytes = _wm_tile_bytes(wc) * (wc.steps if wc.steps > 0 else 1)
    peaks, peak_src = _peaks()
    cpu = None
    if not args.no_cpu:
        from oracle import jepa_oracle as orc
        W = orc.weights_f64([t for t in table if t.name.startswith(("pred.", "enc.proj."))])
        tc = time.perf_counter()
        if wc.steps > 0:
            orc.lewm_rollout(wc, W, st_np[:1], ac_np[:1], wc.steps)
            n_calls = wc.steps
        else:
            orc.lewm_predict(wc, W, st_np[:1], ac_np[:1])
            n_calls = 1
        t_c = time.perf_counter() - tc
        cpu = {"value": n_calls / t_c, "unit": "predictor calls/s", "cores": _oracle_threads(), "kind": "oracle",
               "sample": f"1 candidate, {n_calls} call(s), float64 numpy, timed whole ({t_c * 1e3:.1f} ms)"}
    line = {"metric": "LeWM world-model predictor calls/s on 1 B200", "value": value, "unit": "predictor calls/s",
            "n_gpus": world, "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms_per_step,
            "ms_per_step_min": min(ms_steps), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f16", "data": "synthetic",
            "config": {"workload": wc.name, "candidates": C, "frames": wc.frames, "rollout_steps": wc.steps,
                       "window": wc.window, "dim": wc.dim, "depth": wc.depth, "weights": wc.weights,
                       "ctas": ctas, "l2": "flushed between steps (256 MiB write)"},
            "us_per_call_per_candidate_group": ms_per_step * 1e3 / (wc.steps if wc.steps > 0 else 1),
            "tflops": fl / (ms_per_step / 1000.0) / 1e12,
            "weight_stream": {"bytes_per_cta": tile_bytes, "gbs_per_cta": tile_bytes / (ms_per_step / 1000.0) / 1e9},
            "cpu_baseline": cpu, "gpu_launches": launches, "clocks": clocks,
            "when": datetime.datetime.now(datetime.timezone.utc).strftime("%Y-%m-%dT%H:%M:%S.%fZ")}
    del peaks, peak_src
    print(json.dumps(line), flush=True)
    model.close()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    choices=sorted(synth.WORKLOADS) + sorted(synth.PREDICTORS) + sorted(synth.WORLD_MODELS))
    ap.add_argument("--no-cpu", action="store_true", help="skip the oracle cpu_baseline leg")
    ap.add_argument("--clock-log", default=None,
                    help="CSV of the nvidia-smi clock samples taken during the timed region ({rank} is replaced)")
    ap.add_argument("--quant-f16-copy", action="store_true",
                    help="q8_0 / q4_0 workloads: also keep an f16 copy of the matrices for the large GEMMs")
    ap.add_argument("--forward-only", action="store_true",
                    help="run warm-up + --steps forwards and exit (no timing, no JSON): for ncu launch lists")
    args = ap.parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.workload in synth.PREDICTORS:
        if args.impl == "reference" or world > 1:
            print(json.dumps({"impl": args.impl, "unavailable": "the predictor workload runs on one GPU, ours only"}))
            return 0
        return run_predictor(args, synth.PREDICTORS[args.workload], rank, world, local_rank)
    if args.workload in synth.WORLD_MODELS:
        if args.impl == "reference" or world > 1:
            print(json.dumps({"impl": args.impl, "unavailable": "the world-model workload runs on one GPU, ours only"}))
            return 0
        return run_world_model(args, synth.WORLD_MODELS[args.workload], rank, world, local_rank)
    cfg = synth.WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, cfg, rank, world)
    if world > 1:
        import torch
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        return run_ours(args, cfg, rank, world, local_rank)
    finally:
        if world > 1:
            import torch
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
