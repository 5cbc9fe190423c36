#!/usr/bin/env python3
"""Throughput of the forward + loss of the nanochat GPT block stack on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config d20] [--impl ours|reference]

One step = one whole forward + loss (fp32 -> bf16 weight cast, embedding, all
blocks, lm_head, soft-capped cross-entropy) over one [B, T] batch of synthetic
tokens, on each rank.  With N > 1 (torchrun, one process per GPU) each rank
runs its own batch shard (weak scaling, weights replicated) and the global mean
loss is formed by one all-reduce of (loss sum, token count) per step.

Prints one JSON line (rank 0).  ``value`` is device-timed tokens/s over all
ranks (CUDA events, max over ranks) with inputs resident in HBM; ``e2e`` is the
same metric through the public API with the tokens copied from pinned host
memory and the loss read back every step; ``roofline`` is the dominant kernel
(the tcgen05 projection GEMM) timed per launch with CUDA events on the forward's
stream inside the timed region; ``cpu_baseline`` is the fp64 oracle on a bounded
sample, timed on the host cores.  ``--impl reference`` times that oracle alone.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from workloads import SHAPES, TOKEN_SEED, make_extras, make_tokens, make_weights  # noqa: E402

METRIC = "forward+loss tokens/sec at d20 (1×B200); % of bf16 dense tensor peak"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
DTYPE_NOTE = ("f16 tensor-core operands (weights rounded fp32->bf16 as the method casts them, "
              "held exactly in f16; activations f16), fp32 accumulation, fp32 residual/softmax/loss")
DTYPE_NOTE_BF16 = ("bf16 tensor-core operands (weights rounded fp32->bf16 as the method casts them; "
                   "activations bf16, the pages' compute dtype), fp32 accumulation, fp32 residual/softmax/loss")
DTYPE_NOTE_FP8 = ("e4m3 tensor-core operands with dynamic tensorwise scales for the {what} "
                  "(activations quantised from f16, weights from fp32), fp32 accumulation; other products "
                  "f16; fp32 residual/softmax/loss")
GEMM_KINDS = ("gemm_qkv", "gemm_attn_proj", "gemm_fc", "gemm_mlp_proj", "gemm_lm_head")
ROOFLINE_KIND = "gemm_fc"  # the kind with the largest share of the step
# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one c_fc launch of
# the d20 workload at B=32, T=2048, from an ncu capture of the current kernel
# (CTA pairs, 256x256 tiles) at B=8 scaled to B=32 by the tokens processed:
# reads 55.11 MB = A (41.9 MB, x4) + W (13.1 MB, once); writes 119.29 MB of the
# 167.8 MB output, the other 48.5 MB still dirty in L2 when the kernel ends
# (671.1 - 48.5 MB at B=32).  Valid for that workload and kernel only.
FC_TRAFFIC = {("d20", 32, 2048): (4 * 41.94e6 + 13.11e6) + (4 * 167.77e6 - 48.48e6)}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_work(s, kind):
    """Algorithmic FLOPs (GEMM/attention) or bytes (bandwidth-bound kernels) of one
    launch of `kind` in the forward of workload `s` (per-layer kinds: one layer)."""
    M = s.batch * s.seq_len
    C, H, Hkv, D, V = s.d_model, s.n_head, s.n_kv_head, s.head_dim, s.vocab
    if kind == "gemm_qkv":
        return 2.0 * M * C * (H + 2 * Hkv) * D
    if kind == "gemm_attn_proj":
        return 2.0 * M * H * D * C
    if kind in ("gemm_fc", "gemm_mlp_proj"):
        return 8.0 * M * C * C
    if kind == "gemm_lm_head":
        return 2.0 * M * C * V
    if kind == "rmsnorm":  # fp32 read + bf16 write
        return M * C * 6.0
    if kind == "rope_qknorm":  # bf16 read + write of q and k, table read
        return M * (H + Hkv) * D * 4.0
    if kind == "embedding":
        return M * C * 8.0 + M * 4.0
    if kind == "cast":
        L = s.n_layer
        n = L * (C * (H + 2 * Hkv) * D + C * H * D + 8 * C * C) + V * C
        return n * 6.0
    if kind == "fp8_quant":  # 16-bit read + e4m3 write (amax folded into the producer), mean of a layer's 4
        return 3.0 * M * (6 * C + H * D) / 4
    return 0.0


def kernels_per_step(n_entries, L, fp8_bits, extras_bits):
    """CUDA kernels one forward launches.  The trace has one entry per step of
    the path.  An activation quantisation is one kernel when its producer
    folded the amax in (norms, attention, the relu^2 epilogue), two when a norm
    that mixes in the residual-stream terms produced it.  The weight pass is
    one cast launch, or two launches per batch of up to 112 e4m3 weight tensors
    plus a cast launch for what stays 16-bit."""
    n = n_entries
    if fp8_bits:
        unfused = 0
        if fp8_bits & 1:
            if extras_bits & 4:
                unfused += L  # every first norm mixes in x0
            elif extras_bits & 8:
                unfused += 1  # the norm that keeps x_mid
        if (fp8_bits & 2) and (extras_bits & 8):
            unfused += 1  # the final norm subtracts x_mid
        nq = (6 * L if fp8_bits & 1 else 0) + (1 if fp8_bits & 2 else 0)
        cast_kernels = 2 * ((nq + 111) // 112) + (0 if (fp8_bits & 1 and fp8_bits & 2) else 1)
        n += unfused + cast_kernels - 1
    return n


def train_extra_kernels(L, n_ve, extras_bits):
    """Kernels the further terms add to one training micro-step (the trace
    does not record them): the backout product dlambda = -sum dx . x_mid, one
    value-embedding backward per layer that has a table, per layer the
    lambda products and the mix that carries dx to the block's input (and to
    x0, added back once at the end), and the smear backward (token and gate
    passes).  The forward's terms ride in kernels it launches anyway."""
    n = 0
    if extras_bits & 8:
        n += 1
    if extras_bits & 2:
        n += n_ve
    if extras_bits & 4:
        n += 2 * L + 1
    elif extras_bits & 8:
        n += 1  # the mix at the middle block
    if extras_bits & 1:
        n += 2
    return n


class ClockSampler:
    """nvidia-smi clocks/throttle reasons sampled every 200 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu_index = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        try:
            with open(self.path) as f:
                for line in f:
                    parts = [p.strip() for p in line.split(",")]
                    if len(parts) >= 9:
                        rows.append(parts)
        except OSError:
            pass
        finally:
            try:
                os.unlink(self.path)
            except OSError:
                pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def oracle_sample(s, prefix, seed=TOKEN_SEED, weights=None, extras=None, fp8=None):
    """Runs the fp64 oracle on batch row 0, first `prefix` positions (with the
    full-nanochat terms when `extras` is given); returns (tokens processed,
    seconds)."""
    import oracle
    w = make_weights(s) if weights is None else weights
    x, y = make_tokens(s, seed=seed)
    cfg = oracle.OracleConfig(s.n_layer, s.d_model, s.n_head, s.n_kv_head, s.head_dim, s.seq_len,
                              s.vocab, short_window=s.short_window)
    t0 = time.perf_counter()
    oracle.forward(cfg, w, x[:1, :prefix], y[:1, :prefix], want_logits=False, extras=extras, fp8=fp8)
    return prefix, time.perf_counter() - t0


def _extras_for(s, nc=None):
    """Seeded weights of the full-nanochat terms, value-embedding tables only for
    the layers the library uses them on (nc given) or for every layer."""
    if nc is None:
        return make_extras(s)
    cfg = nc.make_config(s.n_layer, s.d_model, s.n_head, s.n_kv_head, s.head_dim, s.seq_len, s.vocab,
                         s.short_window)
    return make_extras(s, layers=[l for l in range(s.n_layer) if nc.layer_value_embed(cfg, l) == 1])


def run_reference(args, s):
    """The oracle arm: rank 0 times the fp64 CPU oracle; other ranks exit."""
    if int(os.environ.get("RANK", "0")) != 0:
        return
    prefix = args.ref_prefix
    w = make_weights(s)
    ex = _extras_for(s) if args.extras == "all" else None
    f8 = None if args.fp8 == "none" else args.fp8
    for _ in range(args.warmup):
        oracle_sample(s, prefix, weights=w, extras=ex, fp8=f8)
    times = [oracle_sample(s, prefix, weights=w, extras=ex, fp8=f8)[1] for _ in range(args.steps)]
    sec = sum(times) / len(times)
    value = prefix / sec
    sample = f"{s.name} batch row 0, first {prefix} positions, forward+loss per step"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": s.name + ("+extras" if ex else "") + ({None: "", "block": "+fp8block",
                                                                       "all": "+fp8"}[f8]),
                   "global_batch": 1, "seq_len": prefix,
                   "parallelism": "none"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_ours(args, s):
    import torch
    import torch.distributed as dist

    import decoder_only_transformer_nc_b200 as nc
    from decoder_only_transformer_nc_b200 import dp

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", device_id=dev, timeout=timedelta(seconds=120))

    bits = nc.EXTRA_ALL if args.extras == "all" else 0
    fp8_bits = {"none": 0, "block": nc.FP8_BLOCK, "all": nc.FP8_ALL}[args.fp8]
    act = nc.BF16 if args.act_dtype == "bf16" else nc.F16
    cfg = nc.make_config(s.n_layer, s.d_model, s.n_head, s.n_kv_head, s.head_dim, s.seq_len, s.vocab,
                         s.short_window, extras=bits, fp8=fp8_bits, act_dtype=act)
    weights = make_weights(s)
    extras = _extras_for(s, nc) if bits else None
    model = nc.Model.from_numpy(cfg, weights, device=dev, extras=extras)
    B, T = s.batch, s.seq_len
    x, y = make_tokens(s, seed=dp.shard_seed(TOKEN_SEED, rank))
    tx, ty = torch.from_numpy(x).to(dev), torch.from_numpy(y).to(dev)
    ws = torch.empty(nc.workspace_bytes(cfg, B, T), dtype=torch.uint8, device=dev)
    out = {"loss": torch.empty((), dtype=torch.float32, device=dev)}
    red = torch.zeros(2, dtype=torch.float64, device=dev)
    n_valid = float((y != -1).sum())

    def step(trace=None, toks=tx, tgts=ty):
        nc.forward(model, toks, tgts, workspace=ws, out=out, trace=trace)
        if world > 1:
            dp.reduce_loss_into(red, out["loss"], n_valid)

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])

    # warm-up (untimed)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    status = nc.get_status(ws)
    if status != 0:
        raise SystemExit(f"device status after warm-up: {nc.STATUS_NAMES.get(status, status)}")

    probe = nc.LaunchTrace(4)
    try:
        nc.forward(model, tx, ty, workspace=ws, out=out, trace=probe)
    except nc.NcError:
        pass
    n_launch = probe.struct.count
    probe.close()
    torch.cuda.synchronize()
    traces = [nc.LaunchTrace(n_launch) for _ in range(args.steps)]

    stream = torch.cuda.current_stream()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        t0.record(stream)
        for k in range(args.steps):
            step(traces[k])
        t1.record(stream)
        torch.cuda.synchronize()
    barrier()
    ms = t0.elapsed_time(t1) / args.steps
    status = nc.get_status(ws)
    clk = clocks.summary()

    # per-kind launch times from the events of the timed region
    per_kind = {}
    for tr in traces:
        for kind, kms in tr.launches():
            d = per_kind.setdefault(kind, [0.0, 0])
            d[0] += kms
            d[1] += 1
    for tr in traces:
        tr.close()

    # ---- e2e through the public API: pinned host inputs in, loss out, every step
    hx = torch.from_numpy(x).pin_memory()
    hy = torch.from_numpy(y).pin_memory()
    dx, dy = torch.empty_like(tx), torch.empty_like(ty)
    hloss = torch.empty((), dtype=torch.float32).pin_memory()
    for _ in range(2):
        dx.copy_(hx, non_blocking=True)
        dy.copy_(hy, non_blocking=True)
        step(toks=dx, tgts=dy)
        hloss.copy_(out["loss"], non_blocking=True)
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        dx.copy_(hx, non_blocking=True)
        dy.copy_(hy, non_blocking=True)
        step(toks=dx, tgts=dy)
        hloss.copy_(out["loss"], non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = e0.elapsed_time(e1) / args.steps

    # max over ranks
    if world > 1:
        tt = torch.tensor([ms, e2e_ms], dtype=torch.float64, device=dev)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        ms, e2e_ms = float(tt[0]), float(tt[1])

    tokens_all = world * B * T
    value = tokens_all / (ms / 1e3)
    e2e_value = tokens_all / (e2e_ms / 1e3)
    flops = nc.forward_flops(cfg, B, T)
    peaks, peak_src = load_peaks()

    rk_ms, rk_n = per_kind.get(ROOFLINE_KIND, [0.0, 0])
    rk_achieved = kernel_work(s, ROOFLINE_KIND) * rk_n / (rk_ms / 1e3) / 1e12 if rk_ms > 0 else 0.0
    gemm_ms = sum(per_kind[k][0] for k in GEMM_KINDS if k in per_kind)
    gemm_launches = sum(per_kind[k][1] for k in GEMM_KINDS if k in per_kind)
    gemm_flops = sum(kernel_work(s, k) * per_kind[k][1] for k in GEMM_KINDS if k in per_kind)
    achieved = gemm_flops / (gemm_ms / 1e3) / 1e12 if gemm_ms > 0 else 0.0
    peak = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    peak16 = peak
    if fp8_bits:  # e4m3 products: the measured bf16 peak x the nominal e4m3/bf16 ratio 4.5 / 2.25
        peak = 2.0 * peak
    total_traced = sum(v[0] for v in per_kind.values())
    attn_flops_step = flops - sum(kernel_work(s, g) * per_kind[g][1] / args.steps
                                  for g in GEMM_KINDS if g in per_kind)
    kernels = {}
    for k, (kms, n) in sorted(per_kind.items(), key=lambda kv: -kv[1][0]):
        ent = {"launches": n, "ms_total": round(kms, 3), "share": round(kms / total_traced, 4)}
        if k.startswith("gemm"):
            ent["tflops"] = round(kernel_work(s, k) * n / (kms / 1e3) / 1e12, 1)
            if fp8_bits and (k != "gemm_lm_head" or fp8_bits & 2):
                ent["precision"] = "e4m3"
        elif k == "attention":
            ent["tflops"] = round(attn_flops_step * args.steps / (kms / 1e3) / 1e12, 1)
        elif kernel_work(s, k) > 0:
            ent["gbs"] = round(kernel_work(s, k) * n / (kms / 1e3) / 1e9, 1)
        kernels[k] = ent

    result = None
    if rank == 0:
        tflops = flops * world / (ms / 1e3) / 1e12
        burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
        result = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None,
            "dtype": (DTYPE_NOTE if act == nc.F16 else DTYPE_NOTE_BF16) if not fp8_bits else DTYPE_NOTE_FP8.format(
                what="six block projections" + (" and the LM head" if fp8_bits & 2 else "")),
            "data": "synthetic",
            "config": {"workload": s.name + ("+extras" if bits else "") + ({0: "", 1: "+fp8block", 3: "+fp8"}[fp8_bits])
                                   + ("+bf16act" if act == nc.BF16 else ""),
                       "global_batch": world * B, "seq_len": T,
                       "parallelism": f"dp{world}" if world > 1 else "none",
                       "layers": s.n_layer, "d_model": s.d_model,
                       "l2": "inputs larger than L2 (fp32 weights %.2f GB, residual stream %.2f GB per step)"
                             % (4 * sum(a.size for a in _flat(weights)) / 1e9, 4 * B * T * s.d_model / 1e9)},
            "tflops": round(tflops, 1),
            # burst / sustained: MEASURED_PEAKS.json's figures, else the fallback ones ("source")
            "pct_of_bf16_peak": {"burst": round(100 * tflops / world / burst, 2),
                                 "sustained": round(100 * tflops / world / peak16, 2),
                                 "burst_tflops": burst, "sustained_tflops": peak16,
                                 "datasheet_dense_2250": round(100 * tflops / world / 2250.0, 2),
                                 "source": peak_src},
            "roofline": {"kernel": "gemm_kernel<EPI_RELU2_16> (c_fc + ReLU^2: M=B*T, N=4C, K=C)",
                         "bound": "tensor", "achieved": round(rk_achieved, 1),
                         "peak": peak,
                         "peak_kind": (f"bf16_tflops_sustained ({peak_src}); f16 operands, same nominal rate"
                                       if not fp8_bits else
                                       f"2 x bf16_tflops_sustained ({peak_src}): e4m3 operands, nominal "
                                       "e4m3/bf16 dense ratio 4.5/2.25"),
                         "unit": "TFLOP/s", "frac": round(rk_achieved / peak, 4),
                         "traffic": (None if fp8_bits or act == nc.BF16 or (s.name, B, T) not in FC_TRAFFIC
                                     else round(FC_TRAFFIC[(s.name, B, T)])),
                         "traffic_note": (None if fp8_bits or act == nc.BF16 or (s.name, B, T) not in FC_TRAFFIC
                                          else "DRAM bytes of one launch: ncu capture of this kernel at B=8, "
                                               "scaled to B=32 by the tokens processed"),
                         "algorithmic_bytes": (1 if fp8_bits else 2) * (B * T * s.d_model
                                                                         + 4 * s.d_model * s.d_model)
                                              + 2 * 4 * B * T * s.d_model,
                         "launches": rk_n, "avg_launch_ms": round(rk_ms / max(1, rk_n), 4)},
            "gemm_family": {"kernel": "gemm_kernel, all projections (qkv, attn c_proj, c_fc, mlp c_proj, lm_head)",
                            "achieved": round(achieved, 1), "frac": round(achieved / peak, 4),
                            "launches": gemm_launches},
            "kernels": kernels,
            "gpu_launches": kernels_per_step(n_launch, s.n_layer, fp8_bits, bits) * args.steps,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": int(x.nbytes + y.nbytes),
                    "d2h_bytes_per_step": 4},
            "clocks": clk,
            "device_status": nc.STATUS_NAMES.get(status, status),
        }
    if world > 1:
        dist.barrier(device_ids=[local])
        dist.destroy_process_group()
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            del model, ws
            torch.cuda.empty_cache()
            fp8_mode = {0: None, 1: "block", 3: "all"}[fp8_bits]
            n_tok, sec = oracle_sample(s, args.cpu_prefix, weights=weights, extras=extras, fp8=fp8_mode)
            result["cpu_baseline"] = {
                "value": n_tok / sec, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                "sample": f"{s.name} batch row 0, first {args.cpu_prefix} positions, fp64 forward+loss "
                          f"({sec:.1f} s)"}
        print(json.dumps(result), flush=True)


def decode_bytes(s, B, pos):
    """Algorithmic HBM bytes of one decode step at position `pos`: every 16-bit
    projection weight once, the fp32 embedding rows, each layer's visible cached
    K and V rows, and the new position's K and V written."""
    C, H, Hkv, D, V, L = s.d_model, s.n_head, s.n_kv_head, s.head_dim, s.vocab, s.n_layer
    weights = 2 * (L * (C * (H + 2 * Hkv) * D + H * D * C + 8 * C * C) + V * C)
    kv_row = 2 * Hkv * D * 2
    keys = 0
    for l in range(L):
        W = s.seq_len if (l % 4 == 3 or l == L - 1) else s.short_window
        keys += min(pos + 1, W)
    return weights + B * C * 4 + B * kv_row * keys + L * B * kv_row


def run_decode(args, s):
    """KV-cache decode throughput: prefill `--prompt` tokens (untimed), then time
    `--steps` single-position steps for all B rows."""
    import torch

    import decoder_only_transformer_nc_b200 as nc

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", device_id=dev, timeout=timedelta(seconds=120))
    B, T0 = s.batch, args.prompt
    K, Wm = args.steps, args.warmup
    T_max = T0 + Wm + 2 * K + 4
    if T_max > s.seq_len:
        raise SystemExit(f"prompt + steps exceed seq_len {s.seq_len}")
    cfg = nc.make_config(s.n_layer, s.d_model, s.n_head, s.n_kv_head, s.head_dim, s.seq_len, s.vocab,
                         s.short_window)
    model = nc.Model.from_numpy(cfg, make_weights(s), device=dev)
    from decoder_only_transformer_nc_b200 import dp
    x, _ = make_tokens(s, seed=dp.shard_seed(TOKEN_SEED, rank), seq_len=T_max)
    tx = torch.from_numpy(x).to(dev)
    sess = nc.Session(model, B, T_max, device=dev)
    sess.prefill(tx[:, :T0].contiguous())
    logits = torch.empty((B, s.vocab), dtype=torch.float32, device=dev)
    steps_tok = [tx[:, T0 + k].contiguous() for k in range(Wm + 2 * K)]
    # the step captured once in a CUDA graph (position in device memory), or eager launches
    step = (lambda tok: sess.decode_graph(tok)) if args.graph else (lambda tok: sess.decode(tok, logits=logits))
    for k in range(Wm):
        step(steps_tok[k])
    torch.cuda.synchronize()
    if sess.status() != 0:
        raise SystemExit(f"device status after warm-up: {sess.status()}")

    def barrier():
        if world > 1:
            torch.distributed.barrier(device_ids=[local])

    stream = torch.cuda.current_stream()
    pos0 = sess.pos
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        t0.record(stream)
        for k in range(K):
            step(steps_tok[Wm + k])
        t1.record(stream)
        torch.cuda.synchronize()
    barrier()
    ms = t0.elapsed_time(t1) / K
    # e2e: tokens from pinned host memory in, the step's logits out, every step
    hx = torch.from_numpy(x).pin_memory()
    hlog = torch.empty((B, s.vocab), dtype=torch.float32).pin_memory()
    dtok = torch.empty(B, dtype=torch.int32, device=dev)
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for k in range(K):
        dtok.copy_(hx[:, sess.pos], non_blocking=True)
        out = step(dtok)
        hlog.copy_(out, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = e0.elapsed_time(e1) / K
    if world > 1:
        tt = torch.tensor([ms, e2e_ms], dtype=torch.float64, device=dev)
        torch.distributed.all_reduce(tt, op=torch.distributed.ReduceOp.MAX)
        ms, e2e_ms = float(tt[0]), float(tt[1])
    byts = sum(decode_bytes(s, B, pos0 + k) for k in range(K)) / K
    peaks, peak_src = load_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    achieved = byts / (ms / 1e3) / 1e9
    if rank == 0:
        print(json.dumps({
            "metric": "decode tokens/sec (KV cache, one position per row per step)", "value": world * B / (ms / 1e3),
            "unit": UNIT, "n_gpus": world, "steps": K, "warmup": Wm, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": DTYPE_NOTE, "data": "synthetic",
            "config": {"workload": f"{s.name} decode", "global_batch": world * B, "prompt": T0,
                       "launch": "one CUDA graph per step" if args.graph else "eager launches",
                       "positions": [pos0, pos0 + K - 1], "parallelism": f"dp{world}" if world > 1 else "none",
                       "l2": "weights (0.87 GB 16-bit) and KV cache larger than L2"},
            "roofline": {"kernel": "whole decode step (weights + cached K/V streamed once)", "bound": "hbm",
                         "achieved": round(achieved, 1), "peak": hbm, "peak_kind": f"hbm_gbs ({peak_src})",
                         "unit": "GB/s", "frac": round(achieved / hbm, 4), "traffic": None,
                         "algorithmic_bytes": int(byts)},
            "gpu_launches": (3 + 10 * s.n_layer) * K,  # embedding; 10 per layer; final norm, lm_head
            "e2e": {"value": world * B / (e2e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": B * 4,
                    "d2h_bytes_per_step": B * s.vocab * 4},
            "clocks": clocks.summary(),
        }), flush=True)
    if world > 1:
        torch.distributed.barrier(device_ids=[local])
        torch.distributed.destroy_process_group()


def run_train(args, s):
    """Training micro-step: forward + loss + backward (gradients of every weight)
    on the workload's [B, T] batch; the optimizer step is out of scope."""
    import torch

    import decoder_only_transformer_nc_b200 as nc
    from decoder_only_transformer_nc_b200 import dp

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", device_id=dev, timeout=timedelta(seconds=120))
    bits = nc.EXTRA_ALL if args.extras == "all" else 0
    cfg = nc.make_config(s.n_layer, s.d_model, s.n_head, s.n_kv_head, s.head_dim, s.seq_len, s.vocab,
                         s.short_window, extras=bits)
    weights = make_weights(s)
    model = nc.Model.from_numpy(cfg, weights, device=dev, extras=_extras_for(s, nc) if bits else None)
    n_ve = sum(nc.layer_value_embed(cfg, l) == 1 for l in range(s.n_layer)) if bits & nc.EXTRA_VALUE_EMBED else 0
    B, T = s.batch, s.seq_len
    x, y = make_tokens(s, seed=dp.shard_seed(TOKEN_SEED, rank))
    tx, ty = torch.from_numpy(x).to(dev), torch.from_numpy(y).to(dev)
    ws = torch.empty(nc.train_workspace_bytes(cfg, B, T), dtype=torch.uint8, device=dev)
    loss = torch.empty((), dtype=torch.float32, device=dev)
    # every weight gradient in one flat fp32 bucket; with N > 1 ranks the
    # local-mean gradients become the global mean's by NCCL all-reduces of the
    # bucket's pieces on a side stream, each started once the backward has
    # finished that piece (layer by layer, from the launch trace's events)
    flat, grads = dp.grad_bucket(model.tensors)
    n_valid = float((y != -1).sum())
    n_entries = 12 + 24 * s.n_layer
    reducer = dp.OverlappedGradAverage(model.tensors, flat) if world > 1 else None
    sched = nc.LaunchTrace(n_entries) if world > 1 else None  # for the steps that are not timed per launch

    def step(toks=tx, tgts=ty, trace=None):
        flat.zero_()
        tr = trace if trace is not None else sched
        nc.forward_backward(model, toks, tgts, grads=grads, workspace=ws, loss=loss, trace=tr)
        if reducer is not None:
            reducer.launch(tr, n_valid)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if nc.get_status(ws) != 0:
        raise SystemExit(f"device status after warm-up: {nc.get_status(ws)}")
    traces = [nc.LaunchTrace(n_entries) for _ in range(args.steps)]

    def barrier():
        if world > 1:
            torch.distributed.barrier(device_ids=[local])

    stream = torch.cuda.current_stream()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        t0.record(stream)
        for k in range(args.steps):
            step(trace=traces[k])
        t1.record(stream)
        torch.cuda.synchronize()
    barrier()
    ms = t0.elapsed_time(t1) / args.steps
    per_kind = {}
    for tr in traces:
        for kind, kms in tr.launches():
            d = per_kind.setdefault(kind, [0.0, 0])
            d[0] += kms
            d[1] += 1
        tr.close()
    # e2e: tokens and targets from pinned host memory in, the loss out, every step
    hx, hy = torch.from_numpy(x).pin_memory(), torch.from_numpy(y).pin_memory()
    dx, dy = torch.empty_like(tx), torch.empty_like(ty)
    hloss = torch.empty((), dtype=torch.float32).pin_memory()
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        dx.copy_(hx, non_blocking=True)
        dy.copy_(hy, non_blocking=True)
        step(toks=dx, tgts=dy)
        hloss.copy_(loss, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = e0.elapsed_time(e1) / args.steps
    if world > 1:
        tt = torch.tensor([ms, e2e_ms], dtype=torch.float64, device=dev)
        torch.distributed.all_reduce(tt, op=torch.distributed.ReduceOp.MAX)
        ms, e2e_ms = float(tt[0]), float(tt[1])
    status = nc.get_status(ws)
    fwd_flops = nc.forward_flops(cfg, B, T)
    M = B * T
    C, H, Hkv, D, V = s.d_model, s.n_head, s.n_kv_head, s.head_dim, s.vocab
    proj = 2.0 * M * s.n_layer * (C * (H + 2 * Hkv) * D + H * D * C + 8 * C * C)  # block projections
    head = 2.0 * M * C * V
    attn_fwd = fwd_flops - proj - head
    # algorithmic FLOPs of one launch of each backward kind
    work = {"gemm_dgrad": (proj + head) / (4 * s.n_layer + 1), "gemm_wgrad": (proj + head) / (4 * s.n_layer + 1),
            "ce_bwd": head, "attn_bwd": 2.5 * attn_fwd / s.n_layer}
    peaks, peak_src = load_peaks()
    peak = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    total = sum(v[0] for v in per_kind.values())
    kernels = {}
    for k, (kms, n) in sorted(per_kind.items(), key=lambda kv: -kv[1][0]):
        ent = {"launches": n, "ms_total": round(kms, 3), "share": round(kms / total, 4)}
        if k in work:
            ent["tflops"] = round(work[k] * n / (kms / 1e3) / 1e12, 1)
        kernels[k] = ent
    top = max((k for k in work if k in per_kind), key=lambda k: per_kind[k][0])
    top_ach = work[top] * per_kind[top][1] / (per_kind[top][0] / 1e3) / 1e12
    if rank == 0:
        train_flops = 3.0 * fwd_flops
        print(json.dumps({
            "metric": "forward+backward tokens/sec at d20 (1xB200), training micro-step without the optimizer",
            "value": world * M / (ms / 1e3), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": DTYPE_NOTE, "data": "synthetic",
            "config": {"workload": f"{s.name}{'+extras' if bits else ''} train", "global_batch": world * B,
                       "seq_len": T,
                       "parallelism": (f"dp{world}, the fp32 gradient bucket all-reduced by NCCL in per-layer "
                                       "pieces on a side stream, overlapping the backward"
                                       if world > 1 else "none"),
                       "l2": "inputs larger than L2 (saved activations ~40 GB per step)"},
            "tflops_3x_forward": round(train_flops * world / (ms / 1e3) / 1e12, 1),
            "roofline": {"kernel": top, "bound": "tensor", "achieved": round(top_ach, 1), "peak": peak,
                         "peak_kind": f"bf16_tflops_sustained ({peak_src})", "unit": "TFLOP/s",
                         "frac": round(top_ach / peak, 4), "traffic": None,
                         "launches": per_kind[top][1], "avg_launch_ms": round(per_kind[top][0] / per_kind[top][1], 4)},
            "kernels": kernels,
            # 2 L copies launch no kernel; attention bwd is 3 per layer; the further terms' kernels are untraced
            "gpu_launches": (n_entries + train_extra_kernels(s.n_layer, n_ve, bits)) * args.steps,
            "e2e": {"value": world * M / (e2e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": int(x.nbytes + y.nbytes),
                    "d2h_bytes_per_step": 4},
            "clocks": clocks.summary(),
            "device_status": nc.STATUS_NAMES.get(status, status),
        }), flush=True)
    if world > 1:
        torch.cuda.synchronize()
        sched.close()
        torch.distributed.barrier(device_ids=[local])
        torch.distributed.destroy_process_group()


def _flat(w):
    yield w["wte"]
    yield w["lm_head"]
    for lw in w["layers"]:
        yield from lw.values()


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="d20", choices=sorted(SHAPES))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-prefix", type=int, default=1024,
                    help="positions of batch row 0 in the oracle CPU-baseline sample")
    ap.add_argument("--ref-prefix", type=int, default=256,
                    help="positions of batch row 0 per step of the reference (oracle) arm")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--mode", default="forward", choices=["forward", "decode", "train"],
                    help="decode: KV-cache decode steps after a prefill of --prompt tokens")
    ap.add_argument("--prompt", type=int, default=1024, help="decode mode: prompt length")
    ap.add_argument("--graph", action=argparse.BooleanOptionalAction, default=True,
                    help="decode mode: replay one captured CUDA graph per step (--no-graph: eager launches)")
    ap.add_argument("--act-dtype", default="f16", choices=["f16", "bf16"],
                    help="forward mode: 16-bit activation format (bf16 = the pages' compute dtype)")
    ap.add_argument("--fp8", default="none", choices=["none", "block", "all"],
                    help="forward mode: dynamic tensorwise e4m3 for the block projections "
                         "('block') or for them and the LM head ('all')")
    ap.add_argument("--extras", default="none", choices=["none", "all"],
                    help="all: also run the full nanochat terms (smear, value embeddings, "
                         "residual lambdas + x0, backout)")
    ap.add_argument("--batch", type=int, default=None,
                    help="per-rank batch rows instead of the workload's (small profiler captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    s = SHAPES[args.config]
    if args.batch is not None:
        if args.batch < 1:
            raise SystemExit("--batch must be >= 1")
        s = dataclasses.replace(s, batch=args.batch)
    if args.mode == "train" and args.fp8 != "none":
        raise SystemExit("--mode train: the training step runs on 16-bit operands (no --fp8)")
    if args.impl == "reference":
        run_reference(args, s)
    elif args.mode == "decode":
        run_decode(args, s)
    elif args.mode == "train":
        run_train(args, s)
    else:
        run_ours(args, s)


if __name__ == "__main__":
    main()
