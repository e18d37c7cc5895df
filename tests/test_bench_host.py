"""bench.py's host-side pieces, on the CPU: the algorithmic FLOP count the
roofline divides by, the oracle's timed sample, and the reference arm's line."""
import json
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from jepa_video_encoder_b200 import synth  # noqa: E402
from oracle import jepa_oracle as orc  # noqa: E402


def test_block_causal_pair_count_closed_form():
    """LeVJEPA, 16 slots of 196 patches plus the CLS sink: a patch of slot s
    reads the (s+1)*196 patches of slots <= s; the CLS row reads all N keys."""
    cfg = synth.LEVJEPA_VIT_L
    pf, slots, N = 196, 16, 3137
    pairs = pf * pf * sum(s + 1 for s in range(slots)) + N
    assert pairs == 5_227_713
    fl = bench._flops(cfg)
    assert fl["attention"] == 4.0 * pairs * cfg.dim * cfg.depth
    # against the oracle's own mask table on the same shape
    allow = orc.allowed_keys(cfg.n_patches, cfg.patches_per_slot, cfg.has_cls, cfg.mask)
    assert int(allow.sum()) == pairs
    # bidirectional models count every pair
    v = synth.VJEPA2_LONG
    assert bench._flops(v)["attention"] == 4.0 * v.n_tokens ** 2 * v.dim * v.depth


def test_gemm_flops_per_clip():
    cfg = synth.LEVJEPA_VIT_L
    fl = bench._flops(cfg)
    N, D, M, L = 3137, 1024, 4096, 24
    assert fl["gemm_qkv"] + fl["gemm_out"] + fl["gemm_up"] + fl["gemm_down"] == 2.0 * N * L * (3 * D * D + D * D + 2 * D * M)
    assert fl["patch_embed"] == 2.0 * 3136 * 768 * D


def test_cpu_clip_runs_every_rotary_block(monkeypatch):
    """The cpu_baseline times one whole clip: every block's q and k turned."""
    calls = []
    real = orc.rope

    def counting(x, pos, *a, **k):
        calls.append(x.shape)
        return real(x, pos, *a, **k)

    monkeypatch.setattr(orc, "rope", counting)
    cfg = synth.small_config(synth.VJEPA2_LONG_ROPE)
    s = bench.cpu_oracle_clip(cfg)
    assert s["value"] > 0 and s["kind"] == "oracle" and s["cores"] >= 1
    assert len(calls) == 2 * cfg.depth          # q and k of every block, timed whole
    assert f"all {cfg.depth} blocks" in s["sample"]


def test_reference_arm_line(capsys):
    """A reference step is one block of one clip: ms_per_step is that step's
    measured time (so steps x ms_per_step is the run's length), the rate is
    one clip over its whole forward built from the measured parts."""
    class Args:
        steps, warmup = 3, 1
    cfg = synth.small_config(synth.LEVJEPA_VIT_L, frames=2, batch=1)
    assert bench.run_reference(Args(), cfg, rank=0, world=1) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC
    assert line["unit"] == "tokens/s" and line["higher_is_better"] is True and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    # the clip's forward is longer than depth block steps, never shorter
    assert 1000.0 * cfg.n_tokens / line["value"] >= cfg.depth * line["ms_per_step"]
    assert bench.run_reference(Args(), cfg, rank=1, world=2) == 0     # other ranks do no work
    assert capsys.readouterr().out == ""


def test_source_hash_ignores_comments_not_code():
    """A traffic figure stays tied to the kernel's code: comment and blank-line
    edits keep the hash, any change of code or of a string literal (inline
    PTX lives in string literals) changes it."""
    src = ('// header\n#include "x.h"\n/* a\n   b */\n__global__ void k(int* p) {\n'
           '  asm volatile("add.s32 %0, %0, 1; // x" : "+r"(*p));  // bump\n}\n')
    h = bench.hash_sources([src])
    assert bench.hash_sources([src.replace("// bump", "// incremented by one\n\n")]) == h
    assert bench.hash_sources([src.replace("/* a\n   b */", "")]) == h
    assert bench.hash_sources([src.replace("1;", "2;")]) != h                    # PTX in a literal
    assert bench.hash_sources([src.replace("int* p", "long* p")]) != h
    assert bench.hash_sources([src, ""]) != h                                    # file boundaries count
    assert "//" in bench.code_text(src) and "bump" not in bench.code_text(src)  # '//' inside the literal kept


def test_small_configs_are_whole_patches():
    for base in synth.WORKLOADS.values():
        c = synth.small_config(base)
        assert c.img_h % c.patch == 0 and c.img_w % c.patch == 0 and c.frames % c.tubelet == 0
        assert c.n_patches == (c.frames // c.tubelet) * (c.img_h // c.patch) * (c.img_w // c.patch) > 0


def test_both_arms_report_the_same_config_keys():
    cfg = synth.LEVJEPA_VIT_L
    a = bench.run_config(cfg, 1, l2="flushed")
    b = bench.run_config(cfg, 1, l2="not applicable")
    assert set(a) == set(b) and {k: v for k, v in a.items() if k != "l2"} == {k: v for k, v in b.items() if k != "l2"}
    assert a["workload"] == cfg.name and a["global_batch"] == cfg.batch
    assert bench.run_config(cfg, 4, l2="x")["global_batch"] == 4 * cfg.batch


def test_clock_log_keeps_the_timed_region(tmp_path):
    """Only samples taken inside the timed region count; throttle reasons are
    read per sample; other GPUs' lines are ignored; without any sample inside,
    all of them count and the record says so."""
    import datetime as dt
    base = dt.datetime(2026, 12, 2, 22, 0, 0)
    def line(sec, gpu, sm, reasons=("Not Active",) * 4):
        ts = (base + dt.timedelta(seconds=sec)).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
        return f"{ts}, {gpu}, {sm}, 1965, 700.5, 0x0, " + ", ".join(reasons) + "\n"
    log = tmp_path / "clocks.csv"
    log.write_text(line(0.0, 0, 345) + line(0.5, 0, 1900) + line(0.55, 1, 100) +
                   line(0.6, 0, 1950, ("Not Active", "Not Active", "Not Active", "Active")) +
                   line(0.7, 0, 1965) + line(1.5, 0, 400))
    t0 = (base + dt.timedelta(seconds=0.45)).timestamp()
    t1 = (base + dt.timedelta(seconds=0.75)).timestamp()
    c = bench.parse_clock_log(str(log), 0, t0, t1)
    assert c == {"sm_mhz": 1950.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3,
                 "in_region": True}
    c = bench.parse_clock_log(str(log), 0, t1 + 10, t1 + 20)
    assert c["samples"] == 5 and c["in_region"] is False
    log.write_text("garbled, 0, 1800, 1965, 1, 0x0, Not Active, Not Active, Not Active, Not Active\n")
    c = bench.parse_clock_log(str(log), 0, t0, t1)
    assert c["samples"] == 1 and c["sm_mhz"] == 1800.0 and c["in_region"] is False


def test_world_model_flops_and_tile_stream():
    """The world-model line's FLOP count against a count of the oracle's
    matrix products, and its weight-stream size against the matrices it
    covers (every tile 128 x 64 f16; the adaLN chunks start on tiles)."""
    import bench
    from jepa_video_encoder_b200 import synth
    wc = synth.LEWM_WM_STEP
    D, M, H, A, d = wc.dim, wc.mlp, wc.pred_hidden, wc.action_dim, wc.depth
    for T in (1, 2, 3):
        mats = d * (6 * D * D + 3 * D * D + D * D + 2 * D * M) + D * D + A * D + 2 * D * H
        attn = d * 4 * D * T * (T + 1) // 2
        assert bench._wm_flops_per_call(wc, T) == 2 * T * mats + attn
    tiles = bench._wm_tile_bytes(wc) // 16384
    # D = 192: two 128-row tiles per 192-row chunk, three 64-wide K chunks
    per_block = 6 * 2 * 3 + 5 * 3 + 2 * 3 + 6 * 3 + 2 * 12
    assert tiles == 2 * 3 + d * per_block + 6 * 3 + 2 * 12
    weights = sum(int(np.prod(s)) for n, s, k in synth.world_model_specs(wc)
                  if n.startswith("pred.") and n.endswith("weight") and len(s) == 2 and "action_embed.0" not in n)
    assert weights * 2 <= bench._wm_tile_bytes(wc) <= weights * 2 * 1.3
