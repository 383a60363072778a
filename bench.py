"""Benchmark of the attention core on B200: causal GQA prefill TFLOP/s and decode HBM GB/s.

One step = one pass of the whole hot path over one batch of synthetic input:
  * prefill of the GQA workload (B=2, T=4096, H=32, KV=8, hd=128, causal, RoPE base 5e5):
    RoPE on load, QK^T, mask, online softmax, PV, epilogue;
  * one decode step of the KV-cache workload (batch 64, H=32, KV=8, hd=128, cache lengths
    uniform in [1024, 8192]) and of its MQA variant (KV=1): split-KV partials and the
    log-sum-exp merge;
  * one pass of the bf16 block around the same attention shape (x [2,4096,4096], weights
    resident): the x@Wq, x@Wk, x@Wv projections, the attention core, then ctx@Wo;
  * a chunked prefill: the second 2048 rows of the GQA sequences against a cache of their
    4096 rotated keys (written once, before timing).
``value`` is the prefill TFLOP/s (causal FLOPs counted: 4*B*H*hd*allowed pairs); the decode
GB/s (cache rows read + q + out, per launch pair) ride along under ``decode``, the block's
TFLOP/s (projection FLOPs 2*M*N*K plus the attention's) under ``block``, the chunk's under
``chunk``. Kernels are timed with CUDA events on the stream they
are launched on; L2 is flushed (a 256 MiB memset, outside the timed events) before every
step. ``e2e`` times the same call with the step's inputs copied from pinned host memory and
its output copied back, all inside the timed region.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (launched by torchrun) every rank runs its own replica of the step (the path
shards into independent problems; there is no data-path collective): value = all ranks'
FLOPs / the slowest rank's time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "source": "fallback"}
METRIC = "causal GQA prefill TFLOP/s and decode HBM GB/s on 1 B200, % of roofline"
PREFILL = workloads.GQA
DECODE = workloads.DECODE_GQA
DECODE_MQA = workloads.DECODE_MQA
BLOCK = workloads.GQA_BLOCK
CHUNK = workloads.GQA_CHUNK
LATENT = workloads.LATENT_DECODE
# Algorithmic bytes and launches, stated once (see the design notes):
#   decode bytes = cache rows read (K and V) + q + out; prefill FLOPs = PREFILL.flops.
PREFILL_LAUNCHES = 1
DECODE_LAUNCHES = 2       # split pass + merge, per decode workload
PAGE_SIZE = 16            # rows per page of the paged decode (the KV=8 decode workload, pages shuffled)
BLOCK_LAUNCHES = 5        # three projection GEMMs, the prefill, the output GEMM
CHUNK_LAUNCHES = 1
LATENT_LAUNCHES = 4       # the fold, the split pass, the merge, the value up-projection
FUSED_LAUNCHES = 5        # RoPE table, RMSNorm, QKV GEMM (+ rotation, cache write), prefill, Wo GEMM (+ residual)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        p["source"] = "measured"
        return p
    return dict(PEAKS_FALLBACK)


def csrc_sha256() -> str:
    """Hash of the CUDA sources: DRAM counters taken with other sources are not reported."""
    import hashlib
    d = os.path.join(ROOT, "alibi_rope_tile_b200", "csrc")
    h = hashlib.sha256()
    for f in sorted(os.listdir(d)):
        with open(os.path.join(d, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()


def measured_traffic() -> dict:
    """Per-launch DRAM bytes (read + write) from profiles/traffic.json, or {} when the file
    was written for different kernel sources."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return {}
    with open(path) as f:
        t = json.load(f)
    if t.get("csrc_sha256") != csrc_sha256():
        return {}
    return t.get("per_launch_dram_bytes", {})


def decode_bytes(seqlens, w) -> int:
    rows = int(seqlens.sum())
    elt = 2
    return rows * 2 * w.KV * w.hd * elt + 2 * w.B * w.H * w.hd * elt


def dist_setup(n):
    rank, world = int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1))
    if world != n and n > 1:
        raise SystemExit(f"--gpus {n} but WORLD_SIZE={world}: launch with torchrun")
    if world > 1:
        import datetime
        import torch.distributed as dist
        local = int(os.environ.get("LOCAL_RANK", 0))
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return rank, world


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world, device: str = "cuda") -> float:
    """The largest of the ranks' values (each rank times on its own device)."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_rate(units_per_rank: float, world: int, slowest_ms: float) -> float:
    """Whole-job rate: the units all ranks processed over the slowest rank's time (ms)."""
    return world * units_per_rank / (slowest_ms * 1e-3)


class Clocks:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.idx = device_index
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={device_index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "samples": len(sm),
                "reasons": sorted(reasons)}


def cpu_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_sample_tflops(budget_s: float = 12.0):
    """The fp64 oracle on a bounded sample of the prefill workload, as TFLOP/s of causal
    FLOPs: sequence 0, one key/value group (4 query heads) at a time, all 4096 rows, until
    the time budget is spent (about 1 s per group on 16 cores)."""
    from oracle import attention as A
    w = PREFILL
    q, k, v = workloads.prefill_inputs(w)
    group = w.H // w.KV
    pairs = w.T * (w.T + 1) // 2
    flops = done = 0
    t0 = time.perf_counter()
    for g in range(w.KV):
        if time.perf_counter() - t0 >= budget_s:
            break
        A.attention(q[:1, :, g * group:(g + 1) * group], k[:1, :, g:g + 1], v[:1, :, g:g + 1],
                    rope_base=w.rope_base, causal=True)
        flops += 4 * group * w.hd * pairs
        done += 1
    dt = time.perf_counter() - t0
    sample = (f"GQA prefill, sequence 0, {done} of {w.KV} key/value groups ({done * group} of "
              f"{w.H} query heads), all {w.T} rows, fp64 numpy/OpenBLAS")
    return flops / dt / 1e12, dt, sample


def run_reference(args, rank, world):
    """Reference arm: the fp64 CPU oracle, as it stands, on the host cores (rank 0 only)."""
    if rank != 0:
        return
    per_step = max(2.0, 60.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        oracle_sample_tflops(min(per_step, 3.0))
    vals, secs, sample = [], 0.0, ""
    for _ in range(args.steps):
        v, dt, sample = oracle_sample_tflops(per_step)
        vals.append(v)
        secs += dt
    value = statistics.median(vals)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1000.0 * secs / max(1, args.steps), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": PREFILL.name, "sample": sample},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cpu_cores(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_ours(args, rank, world):
    import alibi_rope_tile_b200 as art
    art.lib()
    dev = torch.cuda.current_device()
    stream = torch.cuda.current_stream()
    w = PREFILL
    do_p, do_d = args.only in ("all", "prefill"), args.only in ("all", "decode")
    do_b = args.only in ("all", "block")
    do_c = args.only in ("all", "chunk")

    q, k, v = workloads.prefill_inputs(w)
    dq, dk, dv = q.cuda(), k.cuda(), v.cuda()
    dout = torch.empty_like(dq)
    decs = []
    paged = None
    lat = None
    if do_d:
        for dw in (DECODE, DECODE_MQA):
            hq, hkc, hvc, hsl, hqp = workloads.decode_inputs(dw)
            decs.append(dict(
                w=dw, bytes=decode_bytes(hsl, dw), hq=hq,
                q=hq.cuda(), kc=hkc.cuda(), vc=hvc.cuda(), sl=hsl.cuda(), qp=hqp.cuda(),
                out=torch.empty(hq.shape, dtype=hq.dtype, device="cuda"),
                ws=torch.empty(art.attn_decode_workspace_size(dw.B, dw.H, dw.KV, dw.hd, dw.Lmax),
                               dtype=torch.uint8, device="cuda")))
            if dw is DECODE:
                # the same cache as a shuffled pool of 16-row pages behind a block table
                mb = dw.Lmax // PAGE_SIZE
                need = [mb] * dw.B  # every slot has a page (those past a length are never read)
                g = torch.Generator().manual_seed(dw.seed + 100)
                order = torch.randperm(sum(need), generator=g)
                table = torch.full((dw.B, mb), -1, dtype=torch.int32)
                at = 0
                for b in range(dw.B):
                    table[b, :need[b]] = order[at:at + need[b]].to(torch.int32)
                    at += need[b]
                kp = torch.zeros(sum(need), PAGE_SIZE, dw.KV, dw.hd, dtype=hkc.dtype, device="cuda")
                vp = torch.zeros_like(kp)
                dtab = table.cuda()
                zero = torch.zeros(dw.B, dtype=torch.int32, device="cuda")
                art.attn_kv_write_paged(decs[-1]["kc"], decs[-1]["vc"], kp, vp, dtab, zero, rope_base=0.0)
                paged = dict(w=dw, bytes=decs[-1]["bytes"], q=decs[-1]["q"], sl=decs[-1]["sl"],
                             qp=decs[-1]["qp"], kp=kp, vp=vp, table=dtab,
                             out=torch.empty_like(decs[-1]["out"]),
                             ws=torch.empty_like(decs[-1]["ws"]))
            del hkc, hvc
        lw = LATENT
        lq, lc, luk, luv, lsl = workloads.latent_inputs(lw)
        lat = dict(w=lw, hq=lq, q=lq.cuda(), c=lc.cuda(), uk=luk.cuda(), uv=luv.cuda(), sl=lsl.cuda(),
                   out=torch.empty(lq.shape, dtype=lq.dtype, device="cuda"),
                   ws=torch.empty(int(art.lib().attn_decode_latent_workspace_size(lw.B, lw.H, lw.hd, lw.dc,
                                                                                  lw.Lmax)),
                                  dtype=torch.uint8, device="cuda"),
                   # algorithmic bytes: each latent row read once, q and out, both weights
                   bytes=int(lsl.sum()) * lw.dc * 2 + 2 * lw.B * lw.H * lw.hd * 2
                   + 2 * lw.H * lw.dc * lw.hd * 2)
        del lc
    blk = None
    if do_b:
        bw = BLOCK
        hx, hW = workloads.block_inputs(bw)
        blk = dict(w=bw, hx=hx, x=hx.cuda(), W={n: t.cuda() for n, t in hW.items()},
                   out=torch.empty(hx.shape, dtype=hx.dtype, device="cuda"),
                   ws=torch.empty(art.attn_block_workspace_size(bw.B, bw.T, bw.d, bw.H, bw.KV, bw.hd,
                                                                 torch.bfloat16),
                                  dtype=torch.uint8, device="cuda"))
        # the same block as a fused pre-norm sub-layer: RMSNorm, one Wqkv, cache write, residual
        fz = dict(gamma=torch.ones(bw.d, dtype=torch.bfloat16, device="cuda"),
                  Wqkv=torch.cat([blk["W"]["Wq"], blk["W"]["Wk"], blk["W"]["Wv"]], dim=1).contiguous(),
                  kc=torch.zeros(bw.B, bw.T, bw.KV, bw.hd, dtype=torch.bfloat16, device="cuda"),
                  out=torch.empty_like(blk["out"]),
                  ws=torch.empty(int(art.lib().attn_block_fused_workspace_size(bw.B, bw.T, bw.d, bw.H, bw.KV,
                                                                               bw.hd)),
                                 dtype=torch.uint8, device="cuda"))
        fz["vc"] = torch.zeros_like(fz["kc"])
        blk["fused"] = fz
        del hW
    chk = None
    if do_c:
        cw = CHUNK
        hcq, hck, hcv = workloads.chunk_inputs(cw)
        ckc = torch.zeros(cw.B, cw.Lmax, cw.KV, cw.hd, dtype=torch.bfloat16, device="cuda")
        cvc = torch.zeros_like(ckc)
        art.attn_kv_write(hck.cuda(), hcv.cuda(), ckc, cvc,
                          torch.zeros(cw.B, dtype=torch.int32, device="cuda"), rope_base=cw.rope_base)
        chk = dict(w=cw, hq=hcq, q=hcq.cuda(), kc=ckc, vc=cvc,
                   sl=torch.full((cw.B,), cw.qpos0 + cw.Tq, dtype=torch.int32, device="cuda"),
                   qp=torch.full((cw.B,), cw.qpos0, dtype=torch.int32, device="cuda"),
                   out=torch.empty(hcq.shape, dtype=hcq.dtype, device="cuda"))
        del hck, hcv
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")

    def prefill():
        if do_p:
            art.attn_prefill(dq, dk, dv, dout, rope_base=w.rope_base, causal=True, window=w.window)

    def decode(d):
        art.attn_decode(d["q"], d["kc"], d["vc"], d["sl"], d["qp"], d["out"], workspace=d["ws"],
                        rope_base=d["w"].rope_base)

    def block():
        if blk is not None:
            bw, W = blk["w"], blk["W"]
            art.attn_block(blk["x"], W["Wq"], W["Wk"], W["Wv"], W["Wo"], blk["out"],
                           workspace=blk["ws"], H=bw.H, KV=bw.KV, rope_base=bw.rope_base,
                           causal=bw.causal, window=bw.window)

    def decode_paged():
        if paged is not None:
            art.attn_decode_paged(paged["q"], paged["kp"], paged["vp"], paged["table"], paged["sl"],
                                  paged["qp"], paged["out"], workspace=paged["ws"],
                                  rope_base=paged["w"].rope_base)

    def block_fused():
        if blk is not None:
            bw, fz = blk["w"], blk["fused"]
            art.attn_block_fused(blk["x"], fz["gamma"], fz["Wqkv"], blk["W"]["Wo"], fz["out"], fz["kc"], fz["vc"],
                                 fz["ws"], H=bw.H, KV=bw.KV, rope_base=bw.rope_base, causal=bw.causal,
                                 window=bw.window)

    def decode_latent():
        if lat is not None:
            art.attn_decode_latent(lat["q"], lat["c"], lat["uk"], lat["uv"], lat["sl"], lat["sl"], lat["out"],
                                   workspace=lat["ws"])

    def chunk():
        if chk is not None:
            art.attn_prefill_chunk(chk["q"], chk["kc"], chk["vc"], chk["sl"], chk["qp"], chk["out"],
                                   rope_base=chk["w"].rope_base)

    for _ in range(max(3, args.warmup)):
        flush.zero_()
        prefill()
        for d in decs:
            decode(d)
        block()
        chunk()
        decode_paged()
        decode_latent()
        block_fused()
    torch.cuda.synchronize()
    art.attn_sync_status()

    nev = 2 + 2 * len(decs) + 10
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(nev)] for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    clocks = Clocks(dev)
    time.sleep(0.3)
    t_begin = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_begin.record(stream)
    for s_ in range(args.steps):
        flush.zero_()
        ev[s_][0].record(stream)
        prefill()
        ev[s_][1].record(stream)
        for n, d in enumerate(decs):
            flush.zero_()
            ev[s_][2 + 2 * n].record(stream)
            decode(d)
            ev[s_][3 + 2 * n].record(stream)
        flush.zero_()
        ev[s_][nev - 10].record(stream)
        block_fused()
        ev[s_][nev - 9].record(stream)
        flush.zero_()
        ev[s_][nev - 8].record(stream)
        decode_latent()
        ev[s_][nev - 7].record(stream)
        flush.zero_()
        ev[s_][nev - 6].record(stream)
        block()
        ev[s_][nev - 5].record(stream)
        flush.zero_()
        ev[s_][nev - 4].record(stream)
        chunk()
        ev[s_][nev - 3].record(stream)
        flush.zero_()
        ev[s_][nev - 2].record(stream)
        decode_paged()
        ev[s_][nev - 1].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    art.attn_sync_status()
    p_tot = max(1e-9, max_over_ranks(sum(ev[s_][0].elapsed_time(ev[s_][1]) for s_ in range(args.steps)), world))
    d_tot = [max(1e-9, max_over_ranks(sum(ev[s_][2 + 2 * n].elapsed_time(ev[s_][3 + 2 * n])
                                          for s_ in range(args.steps)), world))
             for n in range(len(decs))]
    b_tot = max(1e-9, max_over_ranks(sum(ev[s_][nev - 6].elapsed_time(ev[s_][nev - 5])
                                         for s_ in range(args.steps)), world))
    c_tot = max(1e-9, max_over_ranks(sum(ev[s_][nev - 4].elapsed_time(ev[s_][nev - 3])
                                         for s_ in range(args.steps)), world))
    g_tot = max(1e-9, max_over_ranks(sum(ev[s_][nev - 2].elapsed_time(ev[s_][nev - 1])
                                         for s_ in range(args.steps)), world))
    l_tot = max(1e-9, max_over_ranks(sum(ev[s_][nev - 8].elapsed_time(ev[s_][nev - 7])
                                         for s_ in range(args.steps)), world))
    f_tot = max(1e-9, max_over_ranks(sum(ev[s_][nev - 10].elapsed_time(ev[s_][nev - 9])
                                         for s_ in range(args.steps)), world))
    region_ms = max_over_ranks(t_begin.elapsed_time(t_end), world)

    # end to end through the public API: the step's inputs go host (pinned) -> device, the
    # kernels run, the results come back device -> host; all inside the timed region
    hq, hk, hv = q.pin_memory(), k.pin_memory(), v.pin_memory()
    hout = torch.empty(q.shape, dtype=q.dtype).pin_memory()
    hdec = [(d["hq"].pin_memory(), torch.empty(d["hq"].shape, dtype=d["hq"].dtype).pin_memory())
            for d in decs]
    if blk is not None:
        hbx = blk["hx"].pin_memory()
        hbo = torch.empty(blk["hx"].shape, dtype=blk["hx"].dtype).pin_memory()
        hfo = torch.empty(blk["hx"].shape, dtype=blk["hx"].dtype).pin_memory()
    if paged is not None:
        hpo = torch.empty(paged["out"].shape, dtype=paged["out"].dtype).pin_memory()
    if lat is not None:
        hlq = lat["hq"].pin_memory()
        hlo = torch.empty(lat["hq"].shape, dtype=lat["hq"].dtype).pin_memory()
    if chk is not None:
        hcq_p = chk["hq"].pin_memory()
        hco = torch.empty(chk["hq"].shape, dtype=chk["hq"].dtype).pin_memory()

    def e2e_step():
        if do_p:
            dq.copy_(hq, non_blocking=True)
            dk.copy_(hk, non_blocking=True)
            dv.copy_(hv, non_blocking=True)
            prefill()
            hout.copy_(dout, non_blocking=True)
        for d, (hdq, hdo) in zip(decs, hdec):
            d["q"].copy_(hdq, non_blocking=True)
            decode(d)
            hdo.copy_(d["out"], non_blocking=True)
        if blk is not None:
            blk["x"].copy_(hbx, non_blocking=True)
            block()
            hbo.copy_(blk["out"], non_blocking=True)
            block_fused()
            hfo.copy_(blk["fused"]["out"], non_blocking=True)
        if chk is not None:
            chk["q"].copy_(hcq_p, non_blocking=True)
            chunk()
            hco.copy_(chk["out"], non_blocking=True)
        if paged is not None:
            # its query tensor is the KV=8 decode's, already copied in above
            decode_paged()
            hpo.copy_(paged["out"], non_blocking=True)
        if lat is not None:
            lat["q"].copy_(hlq, non_blocking=True)
            decode_latent()
            hlo.copy_(lat["out"], non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)

    if rank != 0:
        return
    if args.only != "all":
        print(json.dumps({"only": args.only, "prefill_ms": p_tot / args.steps,
                          "decode_ms": [t / args.steps for t in d_tot],
                          "block_ms": b_tot / args.steps, "chunk_ms": c_tot / args.steps}), flush=True)
        return
    pk = peaks()
    flops_step = w.flops
    per_launch_ms = p_tot / args.steps
    achieved = flops_step / (per_launch_ms * 1e-3) / 1e12
    traffic = measured_traffic()
    decode_out = {}
    for n, d in enumerate(decs):
        ms = d_tot[n] / args.steps
        gbs = d["bytes"] / (ms * 1e-3) / 1e9
        decode_out[d["w"].name] = {
            "value": aggregate_rate(d["bytes"] * args.steps, world, d_tot[n]) / 1e9, "unit": "GB/s",
            "ms": ms, "bytes": d["bytes"],
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / pk["hbm_gbs"], "traffic": traffic.get(d["w"].name),
                         "peak_source": f"{pk.get('source')} copy"}}
    bw = blk["w"]
    b_ms = b_tot / args.steps
    b_tflops = bw.flops / (b_ms * 1e-3) / 1e12
    # the block's attention has the prefill's shape and flags, so its time is the prefill's
    proj_ms = max(1e-9, b_ms - per_launch_ms)
    proj_tflops = bw.projection_flops / (proj_ms * 1e-3) / 1e12
    block_out = {
        "workload": bw.name, "value": aggregate_rate(bw.flops * args.steps, world, b_tot) / 1e12,
        "unit": "TFLOP/s", "ms": b_ms, "flops": bw.flops, "projection_flops": bw.projection_flops,
        "roofline": {"bound": "tensor", "achieved": b_tflops, "peak": pk["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": b_tflops / pk["bf16_tflops"], "traffic": None,
                     "peak_source": f"{pk.get('source')} burst bf16 dense"},
        "projections_derived": {"tflops": proj_tflops, "ms": proj_ms,
                                "frac": proj_tflops / pk["bf16_tflops"],
                                "how": "block time minus the prefill time of the same shape"}}
    f_ms = f_tot / args.steps
    f_tflops = bw.flops / (f_ms * 1e-3) / 1e12
    block_out["fused"] = {
        "what": "RMSNorm, one QKV GEMM (RoPE and cache write in its epilogue), attention, Wo GEMM + residual",
        "value": aggregate_rate(bw.flops * args.steps, world, f_tot) / 1e12, "unit": "TFLOP/s", "ms": f_ms,
        "roofline": {"bound": "tensor", "achieved": f_tflops, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": f_tflops / pk["bf16_tflops"], "traffic": None,
                     "peak_source": f"{pk.get('source')} burst bf16 dense"}}
    if paged is not None:
        ms = g_tot / args.steps
        gbs = paged["bytes"] / (ms * 1e-3) / 1e9
        decode_out[paged["w"].name + f"_paged{PAGE_SIZE}"] = {
            "value": aggregate_rate(paged["bytes"] * args.steps, world, g_tot) / 1e9, "unit": "GB/s",
            "ms": ms, "bytes": paged["bytes"], "page_size": PAGE_SIZE, "pages": "shuffled",
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / pk["hbm_gbs"],
                         "traffic": traffic.get(paged["w"].name + f"_paged{PAGE_SIZE}"),
                         "peak_source": f"{pk.get('source')} copy"}}
    if lat is not None:
        ms = l_tot / args.steps
        gbs = lat["bytes"] / (ms * 1e-3) / 1e9
        decode_out[lat["w"].name] = {
            "value": aggregate_rate(lat["bytes"] * args.steps, world, l_tot) / 1e9, "unit": "GB/s",
            "ms": ms, "bytes": lat["bytes"],
            "note": "each latent tile is fetched twice (as keys and as values); bytes count it once",
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / pk["hbm_gbs"], "traffic": traffic.get(lat["w"].name),
                         "peak_source": f"{pk.get('source')} copy"}}
    cw = chk["w"]
    c_ms = c_tot / args.steps
    c_tflops = cw.flops / (c_ms * 1e-3) / 1e12
    chunk_out = {
        "workload": cw.name, "value": aggregate_rate(cw.flops * args.steps, world, c_tot) / 1e12,
        "unit": "TFLOP/s", "ms": c_ms, "flops": cw.flops,
        "roofline": {"bound": "tensor", "achieved": c_tflops, "peak": pk["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": c_tflops / pk["bf16_tflops"], "traffic": None,
                     "kernel": "prefill_tc_kernel<128, true>",
                     "peak_source": f"{pk.get('source')} burst bf16 dense"}}
    xb = blk["hx"].numel() * blk["hx"].element_size()
    cb = chk["hq"].numel() * chk["hq"].element_size()
    h2d = sum(t.numel() * t.element_size() for t in (q, k, v)) + sum(
        d["hq"].numel() * d["hq"].element_size() for d in decs) + xb + cb
    d2h = q.numel() * q.element_size() + sum(
        d["hq"].numel() * d["hq"].element_size() for d in decs) + 2 * xb + cb
    if paged is not None:
        d2h += paged["out"].numel() * paged["out"].element_size()
    if lat is not None:
        h2d += lat["hq"].numel() * lat["hq"].element_size()
        d2h += lat["hq"].numel() * lat["hq"].element_size()
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        val, dt, sample = oracle_sample_tflops()
        cpu = {"value": val, "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
               "sample": sample, "seconds": round(dt, 2)}
    line = {
        "metric": METRIC, "value": aggregate_rate(flops_step * args.steps, world, p_tot) / 1e12,
        "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": (p_tot + sum(d_tot) + b_tot + c_tot + g_tot + l_tot + f_tot) / args.steps,
        "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "decode_workloads": [d["w"].name for d in decs],
                   "block_workload": bw.name, "chunk_workload": cw.name,
                   "parallelism": f"replicas{world}",
                   "l2": "flushed: 256 MiB memset before every kernel family, outside the events",
                   "timed_region_ms": region_ms},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": pk["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": achieved / pk["bf16_tflops"],
                     "traffic": traffic.get(w.name), "kernel": "prefill_tc_kernel<128, false>",
                     "peak_source": f"{pk.get('source')} burst bf16 dense"},
        "decode": decode_out,
        "block": block_out,
        "chunk": chunk_out,
        "e2e": {"value": aggregate_rate(flops_step * args.steps, world, e2e_ms) / 1e12,
                "unit": "TFLOP/s", "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                "ms_per_step": e2e_ms / args.steps,
                "note": "prefill FLOPs over the whole step incl. copies, both decodes, the block "
                        "(block weights resident; x in, out back) and the chunk (cache resident; "
                        "its queries in, out back)"},
        "gpu_launches": args.steps * (PREFILL_LAUNCHES + DECODE_LAUNCHES * (len(decs) + 1) + BLOCK_LAUNCHES
                                      + CHUNK_LAUNCHES + LATENT_LAUNCHES + FUSED_LAUNCHES),
        "clocks": clk,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", choices=["all", "prefill", "decode", "block", "chunk"], default="all",
                    help="run one kernel family only (for profiler captures; not a bench line)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    rank, world = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
        else:
            run_ours(args, rank, world)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
