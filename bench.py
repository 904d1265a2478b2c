#!/usr/bin/env python
"""Benchmark of the TurboQuant KV-cache hot path on B200.

One step = the whole hot path over one batch of synthetic input on the
long-context decode workload (batch 8, 8 KV heads x d=128, 32 query heads,
context 131072, 4-bit keys / 3-bit values, WHT rotation):

    tq_quantize_kv(K, 4 bit)   8,388,608 bf16 rows -> packed codes + fp16 norms
    tq_quantize_kv(V, 3 bit)   8,388,608 bf16 rows -> packed codes (lane-grouped
                                order, TQ_FMT_GROUPED) + fp16 norms
    tq_decode_attention         rotated query, logits, softmax, value sum,
                                inverse rotation -> fp32 [8, 32, 128]

``value`` is whole-job tokens*kv-heads per second (batch * ctx * kv_heads
per step, summed over ranks, divided by the max-over-ranks device time).
Inputs (4 GiB of bf16 K/V) exceed the 126 MB L2, so no flush is needed.

``--impl reference`` times the CPU oracle (float64 numpy) on a bounded sample
of the same workload instead.  Multi-GPU (torchrun): each rank runs the full
workload on its own data (weak scaling, no collective on the data path).
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode attention tokens·heads/s and quantize rows/s; achieved HBM GB/s vs ~8 TB/s"
UNIT = "tokens·heads/s"
WORKLOAD = "decode_128k"


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["tq", "reference"], default="tq")
    ap.add_argument("--workload", default=WORKLOAD,
                    help="decode_128k (default), llama8b_32k (quick run), qjl_16k "
                         "(2-bit keys with QJL signs, m = 128), paged_128k (paged cache, "
                         "append + decode) or search_1m (top-k inner-product search)")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload batch (profiling on a smaller case only)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    return ap.parse_args()


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def max_over_ranks(ms, world, device, dist):
    """The slowest rank's device time (every rank calls this, in the same order)."""
    if world <= 1:
        return ms
    import torch
    t = torch.tensor([ms], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(units_per_rank, world, steps, ms):
    """Whole-job throughput: every rank processed units_per_rank per step."""
    return world * units_per_rank * steps / (ms / 1e3)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def _code_only(text):
    """C/C++/CUDA source without comments and whitespace (a comment edit does
    not change the kernel a capture measured)."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c == '"':                                   # string literal: keep as is
            j = i + 1
            while j < n and text[j] != '"':
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    return "".join("".join(out).split())


def kernel_source_hash():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "kv_cache_vector_11_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            h.update(name.encode())
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def ncu_traffic(kernel_key):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel sources; else None."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    ent = d.get(kernel_key)
    if not ent or ent.get("source_hash") != kernel_source_hash():
        return None
    return ent.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i, v in enumerate(r)
                          if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows),
                "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons,
                "samples": len(rows)}


def cpu_threads():
    """Threads the oracle can use: numpy's BLAS pool (its elementwise work is
    single-threaded)."""
    try:
        from threadpoolctl import threadpool_info
        n = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        n = 1
    return int(n)


def cpu_info():
    """Host core count and the oracle's BLAS thread count, both recorded."""
    return {"cores": cpu_threads(), "host_cpus": os.cpu_count(), "blas_threads": cpu_threads()}


TARGET_FRAC_OF_8TBS = 0.70


def rank_seeds(rank):
    """Per-rank input seeds (weak scaling: each rank owns a disjoint batch)."""
    import workloads as W
    return {"k": W.SEED_K + 1000 * rank, "v": W.SEED_V + 1000 * rank, "q": W.SEED_Q + rank}


def oracle_sample(k64, v64, q64, d, kbits, vbits, seed_rot):
    """One oracle pass over one (batch, kv head) slice: quantize K and V, then
    decode every query head of the group.  Returns seconds."""
    import numpy as np
    from oracle import attention as oatt, codebook as ocb, quant as oq, rotation as orot
    t0 = time.perf_counter()
    rot = orot.wht_rotation(d, seed_rot)
    ck, tk = ocb.stored_table(kbits, 32)
    cv, tv = ocb.stored_table(vbits, 32)
    qk = oq.quantize(k64, rot, ck, tk, kbits, 32)
    qv = oq.quantize(v64, rot, cv, tv, vbits, 32)
    ki = oq.unpack(qk["words"], kbits, 32, d)
    vi = oq.unpack(qv["words"], vbits, 32, d)
    oatt.decode(q64, rot, ki, qk["norms"], ck, vi, qv["norms"], cv, 32, 1, k64.shape[0])
    np.asarray(0)
    return time.perf_counter() - t0


def run_reference(args):
    """The oracle, as it stands, on host cores: each step is one bounded
    sample (one (batch, kv head) slice, 16384 tokens) of the workload."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    import workloads as W
    cfg = W.WORKLOADS[args.workload]
    d, kb, vb = cfg["head_dim"], cfg["k_bits"], cfg["v_bits"]
    group = cfg["n_q_heads"] // cfg["n_kv_heads"]
    t_sample = min(16384, cfg["ctx"])
    k64 = W.kv_host(1, 1, t_sample, d, seed=W.SEED_K)
    v64 = W.kv_host(1, 1, t_sample, d, seed=W.SEED_V)
    q64 = W.queries_host(1, group, d)
    for _ in range(args.warmup):
        oracle_sample(k64, v64, q64, d, kb, vb, W.SEED_ROT)
    secs = [oracle_sample(k64, v64, q64, d, kb, vb, W.SEED_ROT) for _ in range(args.steps)]
    total = sum(secs)
    value = t_sample * args.steps / total
    sample = (f"1 of {cfg['batch'] * cfg['n_kv_heads']} (batch, kv-head) slices, {t_sample} of "
              f"{cfg['ctx']} tokens: quantize K ({kb}-bit) and V ({vb}-bit), decode {group} query heads")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload, "batch": cfg["batch"],
                       "n_kv_heads": cfg["n_kv_heads"], "n_q_heads": cfg["n_q_heads"],
                       "ctx": cfg["ctx"], "head_dim": d, "k_bits": kb, "v_bits": vb,
                       "rotation": cfg["rot"], "sample_tokens": t_sample},
            "cpu_baseline": {"value": value, "unit": UNIT, **cpu_info(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def _timed(torch, fn, stream, steps, warmup):
    """Average device ms of fn() over `steps` calls after `warmup` calls."""
    for _ in range(max(warmup, 0)):
        fn()
    torch.cuda.synchronize()
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    s.record(stream)
    for _ in range(steps):
        fn()
    e.record(stream)
    torch.cuda.synchronize()
    return s.elapsed_time(e) / steps


def _timed_flushed(torch, fn, stream, steps, warmup, dev):
    """Average device ms of fn() over `steps` calls after `warmup` calls, for
    inputs that fit in L2: before every call a 256 MiB buffer is written (the
    L2 holds 126 MB), outside the timed interval of that call."""
    flush = torch.empty((256 << 20,), dtype=torch.uint8, device=dev)
    for _ in range(max(warmup, 0)):
        flush.fill_(1)
        fn()
    torch.cuda.synchronize()
    total = 0.0
    for i in range(steps):
        flush.fill_(i & 255)
        s = torch.cuda.Event(enable_timing=True)
        e = torch.cuda.Event(enable_timing=True)
        s.record(stream)
        fn()
        e.record(stream)
        torch.cuda.synchronize()
        total += s.elapsed_time(e)
    del flush
    return total / steps


def _roof_line(nbytes, ms, key):
    peak, kind = load_peaks()
    gbs = nbytes / (ms / 1e3) / 1e9
    return {"bound": "hbm", "achieved": round(gbs, 1), "peak": peak, "unit": "GB/s",
            "frac": round(gbs / peak, 4), "traffic": ncu_traffic(key), "kernel": key,
            "algorithmic_bytes": nbytes, "avg_ms": round(ms, 4), "peak_source": kind,
            "frac_of_8tbs": round(gbs / 8000.0, 4), "meets_target": gbs / 8000.0 >= TARGET_FRAC_OF_8TBS}


def run_next(args):
    """Single-GPU measurements of the rows beyond the graded path: the paged
    decode with append (paged_128k) and the inner-product search (search_1m)."""
    import torch
    import kv_cache_vector_11_b200 as tq
    import workloads as W
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    cfg = dict(W.WORKLOADS[args.workload])
    if args.batch is not None and "batch" in cfg:
        cfg["batch"] = args.batch              # profiling only: a smaller paged workload
    d = cfg["head_dim"]
    rot = tq.Rotation(cfg["rot"], d, d, W.SEED_ROT)
    clocks = ClockSampler(0)
    if args.workload == "search_1m":
        n_db, nq, k, bits = cfg["n_db"], cfg["n_queries"], cfg["k"], cfg["bits"]
        c, t = tq.build_codebook(bits)
        x = W.kv_device(1, 1, n_db, d, seed=W.SEED_K, device=dev)
        db = tq.quantize_kv(rot, bits, c, t, x)
        del x
        q = torch.randn((nq, d), device=dev).to(torch.bfloat16)
        ws = torch.empty((tq.search_workspace_size(nq, n_db, d, k),), dtype=torch.uint8, device=dev)
        fn = lambda: tq.search_topk(rot, bits, c, q, db["codes"], db["norms"], k, workspace=ws,
                                    stream=stream)
        clocks.start()
        ms = _timed_flushed(torch, fn, stream, args.steps, args.warmup, dev)
        clk = clocks.stop()
        row_bytes = tq.code_words_per_row(bits, 32, d) * 4 + 2 * (d // 32)
        nbytes = n_db * row_bytes + q.numel() * 2 + nq * k * 8
        line = {"metric": "inner-product search: database rows x queries scored per second",
                "value": n_db * nq / (ms / 1e3), "unit": "row-queries/s", "n_gpus": 1,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic", "config": {"workload": args.workload, **cfg,
                                                "l2": "database smaller than L2: a 256 MiB buffer is "
                                                      "written before every timed call (outside it)"},
                "roofline": _roof_line(nbytes, ms, "search_qrows_kernel + search_tc_kernel (sample, main) + "
                                       "topk_bound_kernel + topk_lists_kernel" if k <= 16 and d in (64, 128) else
                                       "search_prep_kernel + search_scores_kernel + topk_pass_kernel"),
                "gpu_launches": None, "clocks": clk,
                "note": "algorithmic bytes = the packed database read once, the queries and the "
                        "k results; each 128-row tile is dequantized once into shared memory and "
                        "scored against every query by one tcgen05 MMA, every thread keeps a "
                        "top-k list, and one kernel selects each query's k best of the lists"}
    else:
        B, Hkv, Hq, T = cfg["batch"], cfg["n_kv_heads"], cfg["n_q_heads"], cfg["ctx"]
        kb, vb, P = cfg["k_bits"], cfg["v_bits"], cfg["page_size"]
        kcb, vcb = tq.build_codebook(kb), tq.build_codebook(vb)
        max_pages = T // P
        n_pages = B * max_pages
        g = torch.Generator(device="cpu")
        g.manual_seed(5)
        table = torch.randperm(n_pages, generator=g).to(torch.int32).reshape(B, max_pages).to(dev)
        wk, wv, nb = tq.code_words_per_row(kb, 32, d), tq.code_words_per_row(vb, 32, d), d // 32
        pages = {}
        for name, bits, cb, seed, w in (("k", kb, kcb, W.SEED_K, wk), ("v", vb, vcb, W.SEED_V, wv)):
            x = W.kv_device(B, Hkv, T, d, seed=seed, device=dev)
            xq = tq.quantize_kv(rot, bits, cb[0], cb[1], x)
            del x
            # scatter [b][hk][t] rows into [page][hk][P] through the table
            t_idx = torch.arange(T, device=dev)
            rows = ((table[:, (t_idx // P)].long()[:, None, :] * Hkv +
                     torch.arange(Hkv, device=dev)[None, :, None]) * P + (t_idx % P)[None, None, :])
            pc = torch.empty((n_pages * Hkv * P, w), dtype=torch.int32, device=dev)
            pn = torch.empty((n_pages * Hkv * P, nb), dtype=torch.int16, device=dev)
            pc[rows.reshape(-1)] = xq["codes"]
            pn[rows.reshape(-1)] = xq["norms"]
            del xq
            pages[name + "_codes"] = pc.view(n_pages, Hkv, P, w)
            pages[name + "_norms"] = pn.view(n_pages, Hkv, P, nb)
        q = torch.randn((B, Hq, d), device=dev).to(torch.bfloat16)
        kn = torch.randn((B, Hkv, d), device=dev).to(torch.bfloat16)
        vn = torch.randn((B, Hkv, d), device=dev).to(torch.bfloat16)
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=dev)
        ws = torch.empty((tq.decode_workspace_size(B, Hq, Hkv, T, d),), dtype=torch.uint8, device=dev)
        fn = lambda: tq.decode_append_paged(rot, kb, vb, kcb, vcb, q, kn, vn, pages, table, Hkv, T,
                                            P, out=out, workspace=ws, stream=stream)
        clocks.start()
        ms = _timed(torch, fn, stream, args.steps, args.warmup)
        clk = clocks.stop()
        rows_all = B * Hkv * T
        nbytes = (rows_all * (4 * wk + 4 * wv + 4 * nb) + q.numel() * 2 + out.numel() * 4 +
                  B * Hkv * (2 * 2 * d + 4 * wk + 4 * wv + 4 * nb) + table.numel() * 4)
        line = {"metric": METRIC, "value": rows_all / (ms / 1e3), "unit": UNIT, "n_gpus": 1,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic", "config": {"workload": args.workload, **cfg,
                                                "step": "append the new token's K/V + decode"},
                "roofline": _roof_line(nbytes, ms, f"decode_mma_prep_kernel<{d}> (append) + "
                                                   f"decode_mma_kernel<{d},{kb},{vb},false> (paged)"
                                                   " + decode_combine_kernel"),
                "gpu_launches": 3 * args.steps, "clocks": clk}
    print(json.dumps(line), flush=True)


def run_tq(args):
    import torch
    import torch.distributed as dist

    rank, world, local = dist_env()
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)

    import kv_cache_vector_11_b200 as tq
    import workloads as W

    cfg = dict(W.WORKLOADS[args.workload])
    if args.batch is not None:
        cfg["batch"] = args.batch
    B, Hkv, Hq, T, d = cfg["batch"], cfg["n_kv_heads"], cfg["n_q_heads"], cfg["ctx"], cfg["head_dim"]
    kb, vb = cfg["k_bits"], cfg["v_bits"]
    rows = B * Hkv * T

    # per-rank data (weak scaling): seeds offset by rank
    seeds = rank_seeds(rank)
    k = W.kv_device(B, Hkv, T, d, seed=seeds["k"], device=dev)
    v = W.kv_device(B, Hkv, T, d, seed=seeds["v"], device=dev)
    g = torch.Generator(device=dev)
    g.manual_seed(seeds["q"])
    q = torch.randn((B, Hq, d), generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)

    rot = tq.Rotation(cfg["rot"], d, d, W.SEED_ROT)
    ck, tk = tq.build_codebook(kb)
    cv, tv = tq.build_codebook(vb)
    wk, wv = tq.code_words_per_row(kb, 32, d), tq.code_words_per_row(vb, 32, d)
    m = cfg.get("qjl_m")                       # QJL signs on the keys (None: codes only)
    qjl = tq.Rotation("gauss", m, d, W.SEED_QJL) if m else None
    kout = {"codes": torch.empty((rows, wk), dtype=torch.int32, device=dev),
            "norms": torch.empty((rows, d // 32), dtype=torch.int16, device=dev)}
    if m:
        kout["signs"] = torch.empty((rows, m // 32), dtype=torch.int32, device=dev)
        kout["rnorm"] = torch.empty((rows,), dtype=torch.int16, device=dev)
    vout = {"codes": torch.empty((rows, wv), dtype=torch.int32, device=dev),
            "norms": torch.empty((rows, d // 32), dtype=torch.int16, device=dev)}
    out = torch.empty((B, Hq, d), dtype=torch.float32, device=dev)
    ws_bytes = tq.decode_workspace_size(B, Hq, Hkv, T, d)
    ws = torch.empty((max(ws_bytes, 16),), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def quant_k(src=k):
        tq.quantize_kv(rot, kb, ck, tk, src, qjl=qjl, out=kout, stream=stream)

    # the value cache in the lane-grouped code order (d = 128)
    vgrp = d == 128

    def quant_v(src=v):
        tq.quantize_kv(rot, vb, cv, tv, src, out=vout, stream=stream, grouped=vgrp)

    def decode(qq=q):
        tq.decode_attention(rot, kb, vb, ck, cv, qq, kout["codes"], kout["norms"],
                            vout["codes"], vout["norms"], Hkv, T, qjl=qjl,
                            qjl_signs=kout.get("signs"), qjl_rnorm=kout.get("rnorm"),
                            out=out, workspace=ws, stream=stream, v_grouped=vgrp)

    lg = torch.empty((B, Hq, T), dtype=torch.float32, device=dev) if m else None

    def score(qq=q):
        # the QJL workload's third stage: raw scores with the QJL correction
        tq.attn_logits(rot, kb, ck, qq, kout["codes"], kout["norms"], Hkv, T, qjl=qjl,
                       qjl_signs=kout["signs"], qjl_rnorm=kout["rnorm"], logits=lg, stream=stream)

    # the step: quantize K, quantize V, then decode attention; the QJL workload
    # also scores raw logits (its statement asks for logits) before decoding
    tail = [score, decode] if m else [decode]

    def third(qq=q):
        for f in tail:
            f(qq)

    def barrier():
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    for _ in range(max(args.warmup, 0)):
        quant_k(); quant_v(); third()
    barrier()

    K = args.steps
    n_ev = 3 + len(tail)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(K)]
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()
    start.record(stream)
    for i in range(K):
        ev[i][0].record(stream)
        quant_k()
        ev[i][1].record(stream)
        quant_v()
        ev[i][2].record(stream)
        for j, f in enumerate(tail):
            f()
            ev[i][3 + j].record(stream)
    end.record(stream)
    barrier()
    clk = clocks.stop()
    elapsed_ms = start.elapsed_time(end)
    t_qk = [ev[i][0].elapsed_time(ev[i][1]) for i in range(K)]
    t_qv = [ev[i][1].elapsed_time(ev[i][2]) for i in range(K)]
    t_tail = [[ev[i][2 + j].elapsed_time(ev[i][3 + j]) for i in range(K)] for j in range(len(tail))]
    t_dec = t_tail[-1]

    elapsed_ms = max_over_ranks(elapsed_ms, world, dev, dist)

    tokens_heads = B * T * Hkv
    value = weak_scaling_value(tokens_heads, world, K, elapsed_ms)

    # algorithmic bytes per launch
    qjl_bytes = rows * (m // 8 + 2) if m else 0      # sign words + fp16 residual norm per row
    qk_bytes = rows * (2 * d + 4 * wk + 2 * (d // 32)) + qjl_bytes
    qv_bytes = rows * (2 * d + 4 * wv + 2 * (d // 32))
    dec_bytes = rows * (4 * wk + 4 * wv + 4 * (d // 32)) + qjl_bytes + q.numel() * 2 + out.numel() * 4
    # logits: K codes, norms, signs, residual norms read; fp32 scores written
    lg_bytes = rows * (4 * wk + 2 * (d // 32)) + qjl_bytes + q.numel() * 2 + lg.numel() * 4 if m else 0
    peak, peak_kind = load_peaks()
    avg = lambda xs: sum(xs) / len(xs)

    def roof(nbytes, ms, key):
        gbs = nbytes / (ms / 1e3) / 1e9
        traffic = ncu_traffic(key)
        f8 = gbs / 8000.0
        return {"bound": "hbm", "achieved": round(gbs, 1), "peak": peak, "unit": "GB/s",
                "frac": round(gbs / peak, 4), "traffic": traffic, "kernel": key,
                "algorithmic_bytes": nbytes, "avg_ms": round(ms, 4), "peak_source": peak_kind,
                "frac_of_8tbs": round(f8, 4), "meets_target": f8 >= TARGET_FRAC_OF_8TBS}

    roof_qk = roof(qk_bytes, avg(t_qk), f"quantize_qjl_tc_kernel<{d},{kb}>" if m
                   else f"quantize_rot_tc_kernel<{d},{kb},false>")
    grp = ",grouped" if vgrp else ""
    roof_qv = roof(qv_bytes, avg(t_qv), f"quantize_rot_tc_kernel<{d},{vb},false{grp}>")
    roof_dec = roof(dec_bytes, avg(t_dec),
                    f"decode_mma_prep_kernel<{d}> + decode_mma_kernel<{d},{kb},{vb},{'true' if m else 'false'}{grp}>"
                    " + decode_combine_kernel")
    kernels = [roof_qk, roof_qv, roof_dec]
    if m:
        kernels.insert(2, roof(lg_bytes, avg(t_tail[0]), f"logits_mma_kernel<{d},{kb}>"))
    dominant = max(kernels, key=lambda r: r["avg_ms"])

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(torch, tq, k, v, q, quant_k, quant_v, third, out, stream, dev, K, world,
                      tokens_heads, barrier, dist)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not m:
        cpu = run_cpu_baseline(k, v, q, cfg)   # the oracle's sample covers the decode step only

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": elapsed_ms / K, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) x log-normal channel scales, 4 outlier channels x20)",
            "config": {"workload": args.workload, "batch": B, "n_kv_heads": Hkv, "n_q_heads": Hq,
                       "ctx": T, "head_dim": d, "k_bits": kb, "v_bits": vb,
                       "rotation": cfg["rot"], "block": 32, "qjl_m": m,
                       "step": ("quantize K (QJL) + quantize V + raw logits + decode attention" if m
                                else "quantize K + quantize V + decode attention"),
                       "l2": "inputs (4 GiB bf16 K/V) larger than L2; no flush",
                       "v_layout": "grouped" if vgrp else "plain"},
            "quantize_rows_per_s": world * 2 * rows * K / ((sum(t_qk) + sum(t_qv)) / 1e3),
            "decode_tokens_heads_per_s": world * tokens_heads * K / (sum(t_dec) / 1e3),
            "roofline": dominant,
            "roofline_kernels": kernels,
            # quantize K, quantize V, (logits,) decode prep, decode, combine
            "gpu_launches": (6 if m else 5) * K,
            "clocks": clk,
            "e2e": e2e,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_e2e(torch, tq, k, v, q, quant_k, quant_v, decode, out, stream, dev, K, world,
            tokens_heads, barrier, dist):
    """Same step through the public API with pinned HOST inputs: H2D copies of
    K, V and q, the three library calls, and a D2H copy of the output, all
    inside the timed region."""
    steps = max(1, min(K, 3))
    hk = torch.empty(k.shape, dtype=k.dtype, pin_memory=True)
    hv = torch.empty(v.shape, dtype=v.dtype, pin_memory=True)
    hq = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
    ho = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    hk.copy_(k); hv.copy_(v); hq.copy_(q)
    dk = torch.empty_like(k); dv = torch.empty_like(v); dq = torch.empty_like(q)
    barrier()
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    s.record(stream)
    for _ in range(steps):
        dk.copy_(hk, non_blocking=True)
        dv.copy_(hv, non_blocking=True)
        dq.copy_(hq, non_blocking=True)
        quant_k(dk)
        quant_v(dv)
        decode(dq)
        ho.copy_(out, non_blocking=True)
    e.record(stream)
    barrier()
    ms = max_over_ranks(s.elapsed_time(e), world, dev, dist)
    del dk, dv, dq
    return {"value": weak_scaling_value(tokens_heads, world, steps, ms), "unit": UNIT,
            "h2d_bytes_per_step": hk.numel() * 2 + hv.numel() * 2 + hq.numel() * 2,
            "d2h_bytes_per_step": ho.numel() * 4, "steps": steps}


def run_cpu_baseline(k, v, q, cfg):
    """The oracle on the host cores, on the first two (batch 0, kv head) slices
    of the same inputs (all their tokens)."""
    import numpy as np
    d = cfg["head_dim"]
    group = cfg["n_q_heads"] // cfg["n_kv_heads"]
    import workloads as W
    T = cfg["ctx"]
    n_slices = min(2, cfg["n_kv_heads"])
    secs = 0.0
    for h in range(n_slices):
        k64 = k[h * T:(h + 1) * T].float().cpu().numpy().astype(np.float64)
        v64 = v[h * T:(h + 1) * T].float().cpu().numpy().astype(np.float64)
        q64 = q[0:1, h * group:(h + 1) * group].float().cpu().numpy().astype(np.float64)
        secs += oracle_sample(k64, v64, q64, d, cfg["k_bits"], cfg["v_bits"], W.SEED_ROT)
    return {"value": n_slices * T / secs, "unit": UNIT, **cpu_info(), "kind": "oracle",
            "sample": f"batch 0, kv heads 0..{n_slices - 1}, all {T} tokens each: quantize K and V, "
                      f"decode {group} query heads per kv head; {secs:.1f} s"}


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
    elif args.workload in ("paged_128k", "search_1m"):
        run_next(args)
    else:
        run_tq(args)


if __name__ == "__main__":
    main()
