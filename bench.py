"""Benchmark: BF16 decode GB/s of the 8B-shaped weight set on B200, with the
fraction of the HBM roofline and the compressed size as % of BF16.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one full decode of the llama8b_shaped weight set (32 decoder layers
of q/o 4096x4096, k/v 1024x4096, gate/up 14336x4096, down 4096x14336 and two
4096 norms, plus a 128256x4096 embedding and lm_head: 8,030,257,152 BF16
weights, 16.06 GB) by ONE grouped launch (df_decode_batch_run) from the
compressed containers resident in HBM into 16.06 GB of BF16 outputs. The inputs
are far larger than L2, so no L2 flush is needed between steps.

Also reported on the same line: the layer-by-layer decode into one reused
buffer (34 grouped launches per pass), the GPU encode throughput, the
end-to-end number through the public API from pinned host memory (compressed
bytes host->device, decode, BF16 host<-device every step), the roofline of the
decode kernel against the measured HBM copy bandwidth, the CPU oracle timed on
a bounded sample, and the SM clocks sampled during the timed region.

With N > 1 (torchrun), every rank decodes its own copy of the weight set
(weak scaling, no data-path collective); `value` = all ranks' bytes over the
slowest rank's time.

--impl reference times the CPU oracle (the plain single-threaded decoder) on
the host cores on a bounded sample of the same workload, same metric and unit.
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
sys.path.insert(0, ROOT)

L2_BYTES = 126 * 1000 * 1000          # B200 L2
L2_FLUSH_BELOW = 2 * L2_BYTES          # inputs + outputs below this get an L2 flush per step
L2_FLUSH_BYTES = 512 << 20             # the flush buffer (a write larger than L2)

METRIC = "BF16 decode GB/s + % of B200 HBM roofline; compressed size % of BF16"
WORKLOAD = ("llama8b_shaped: 32 Llama-style decoder layers (q/o 4096x4096, k/v 1024x4096, gate/up 14336x4096, "
            "down 4096x14336, 2 RMSNorm 4096) + embedding and lm_head 128256x4096; 8,030,257,152 BF16 weights "
            "(16.06 GB); decoded whole by one grouped launch")
FALLBACK_HBM_GBS = 6650.0


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--e2e-steps", type=int, default=3)
    p.add_argument("--workload", default="llama8b_shaped",
                   choices=["llama8b_shaped", "llama_layer", "single_1024x4096", "heavy_tail_64m", "mixed_2000"],
                   help="weight set to decode (the headline number is llama8b_shaped)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--chunk-bytes", type=int, default=0,
                   help="format chunk size C in bytes (0: 32, or 16 where the shortest code is 1 bit)")
    p.add_argument("--threads-per-block", type=int, default=256, help="format block size T in chunks")
    return p.parse_args()


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        backend = "nccl" if _cuda_ok() else "gloo"
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=600))
    return world, rank, local


def _cuda_ok():
    import torch

    return torch.cuda.is_available()


def max_over_ranks(x: float, world: int, device=None) -> float:
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def measured_hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs: STREAM-style copy)"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback (6.65 TB/s, earlier measurement on this pool)"


class ClockSampler:
    """nvidia-smi SM clocks and throttle reasons, sampled during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        try:
            import tempfile

            fd, self.path = tempfile.mkstemp(prefix=f"df11_clocks_rank{self.index}_", suffix=".csv")
            self.fh = os.fdopen(fd, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(self.index)], stdout=self.fh, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception as e:  # nvidia-smi missing: report no clocks
            log("clock sampling unavailable:", e)
            self.proc = None

    def stop(self) -> dict | None:
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        sm, mx, reasons = [], [], set()
        lines = open(self.path).read().splitlines()
        os.unlink(self.path)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for name, val in zip(names, parts[4:8]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


def source_digest(paths):
    """Digest of the code in `paths` with comments and whitespace removed: a
    comment edit keeps the digest, any change to the code changes it."""
    import re

    h = hashlib.sha256()
    for p in paths:
        with open(p, encoding="utf-8") as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()[:16]


def decode_traffic_record():
    """ncu DRAM bytes per weight for the decode kernel, if captured for the
    current kernel source (profiles/decode_traffic.json)."""
    path = os.path.join(ROOT, "profiles", "decode_traffic.json")
    src = os.path.join(ROOT, "lossless_bf16_weight_huffman_b200", "csrc", "df_decode.cu")
    try:
        rec = json.load(open(path))
    except Exception:
        return None
    if rec.get("kernel_source_sha") != source_digest([src]):
        return None
    return rec


# ---------------------------------------------------------------------------------------------


def run_reference(args, world, rank):
    """The oracle, as it stands, on the host cores: each step decodes a bounded
    sample of the workload (layer 0's q_proj, 16,777,216 weights)."""
    if rank != 0:
        return
    import oracle
    from lossless_bf16_weight_huffman_b200 import synth

    spec = [s for s in synth.llama8b_shaped() if s.name == "layers.0.q_proj"][0]
    w = synth.generate(spec)
    enc = oracle.encode(w)
    for _ in range(args.warmup):
        oracle.decode_encoded(enc)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        out = oracle.decode_encoded(enc)
        times.append(time.perf_counter() - t0)
    assert (out == w).all()
    total = sum(times)
    gbs = 2 * w.size * args.steps / total / 1e9
    line = {
        "metric": METRIC, "value": round(gbs, 4), "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(1e3 * total / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "u8", "data": "synthetic", "impl": "reference",
        "config": {"workload": WORKLOAD, "sample": "layers.0.q_proj (16,777,216 weights) per step",
                   "parallelism": "host, single thread"},
        "compressed_pct": round(100.0 * enc.container_bytes / (2 * w.size), 3),
        "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": "layers.0.q_proj decoded bit-serially, 16,777,216 weights per step"},
        "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def cpu_baseline_sample(specs):
    """The oracle decoder (single thread) on layer 0 of the weight set."""
    import oracle
    from lossless_bf16_weight_huffman_b200 import synth

    layer0 = [s for s in specs if s.name.startswith("layers.0.")]
    if not layer0:  # another weight set: its first tensors, up to ~2e8 weights
        layer0, tot = [], 0
        for s in specs:
            if tot >= 200_000_000:
                break
            layer0.append(s)
            tot += s.numel
    encs = []
    for s in layer0:
        w = synth.generate(s)
        encs.append((w, oracle.encode(w)))
    n = sum(w.size for w, _ in encs)
    t0 = time.perf_counter()
    for w, e in encs:
        out = oracle.decode_encoded(e)
        assert (out == w).all()
    dt = time.perf_counter() - t0
    return {"value": round(2 * n / dt / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"{'layer 0' if layer0[0].name.startswith('layers.0.') else 'first tensors'} of the "
                      f"weight set ({n:,} weights), bit-serial decode, one host thread, "
                      f"{dt:.1f} s"}


def run_gpu(args, world, rank, local):
    import numpy as np
    import torch

    from lossless_bf16_weight_huffman_b200 import api, build, codec, synth

    build.build_all()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    specs = synth.weight_set(args.workload)
    n_total = sum(s.numel for s in specs)
    max_n = max(s.numel for s in specs)

    # ---- generate on the host, copy to HBM, encode on the GPU. The histograms of all
    # tensors run back to back (one timed region), then the host builds every code, then
    # all encodes run back to back (another timed region).
    t_setup = time.time()
    staging = torch.empty(max_n, dtype=torch.int16, pin_memory=True)
    src = []
    for s in specs:
        n = s.numel
        synth.fill_ptr(s, staging.data_ptr(), n)
        x = torch.empty(n, dtype=torch.int16, device=dev)
        x.copy_(staging[:n])
        torch.cuda.synchronize()  # the staging buffer is refilled next
        src.append(x)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    hist_d = torch.empty((len(specs), 256), dtype=torch.int64, device=dev)
    ev[0].record()
    for i, x in enumerate(src):
        api.df_histogram(x, hist_d[i])
    ev[1].record()
    hists = hist_d.cpu().numpy().view(np.uint64)
    plans = []
    for i, (s, x) in enumerate(zip(specs, src)):
        code = api.df_build_code(hists[i], 32)
        C = args.chunk_bytes or codec.auto_chunk_bytes(code)
        TPB = args.threads_per_block
        lut = torch.from_numpy(api.df_build_lut(code).view(np.int32)).to(dev)
        z = api.df_plan(code, hists[i], s.numel, C, TPB).as_dict()
        bufs = dict(stream=torch.empty(z["stream_bytes"], dtype=torch.uint8, device=dev),
                    gaps=torch.empty(z["gap_bytes"], dtype=torch.uint8, device=dev),
                    offsets=torch.empty(z["n_blocks"] + 1, dtype=torch.int64, device=dev),
                    sm=torch.empty(s.numel, dtype=torch.uint8, device=dev))
        plans.append((code, C, TPB, lut, z, bufs))
    ws = torch.empty(max(p[4]["encode_ws_bytes"] for p in plans), dtype=torch.uint8, device=dev)
    torch.cuda.synchronize()
    ev[2].record()
    for x, (code, C, TPB, lut, z, bufs) in zip(src, plans):
        api.df_encode(code, x, z["total_bits"], C, TPB, bufs["stream"], bufs["gaps"], bufs["offsets"], bufs["sm"],
                      ws, err)
    ev[3].record()
    torch.cuda.synchronize()
    hist_ms = ev[0].elapsed_time(ev[1])
    enc_ms = ev[2].elapsed_time(ev[3])
    del ws
    comps = [codec.Compressed(n=s.numel, shape=s.shape, code=code, lut=lut, sizes=z, chunk_bytes=C,
                              threads_per_block=TPB, **bufs)
             for s, (code, C, TPB, lut, z, bufs) in zip(specs, plans)]
    assert api.df_read_error(err) == 0, "encode reported an error"
    container = sum(c.container_bytes for c in comps)
    read_bytes = sum(c.read_bytes() for c in comps)
    log(f"[rank {rank}] setup {time.time() - t_setup:.1f} s: {len(specs)} tensors, {n_total:,} weights, "
        f"container {100 * container / (2 * n_total):.3f}% of BF16")

    # ---- (i) whole-set decode: one grouped launch per step
    outs = [torch.empty(c.n, dtype=torch.int16, device=dev) for c in comps]
    dec = codec.BatchDecoder(comps, outs)
    for _ in range(max(args.warmup, 1)):
        dec.run(err)
    torch.cuda.synchronize()
    assert api.df_read_error(err) == 0, "decode reported an error"
    for x, o, s in zip(src, outs, specs):
        if not torch.equal(x, o):
            raise SystemExit(f"decode mismatch on {s.name}")
    log(f"[rank {rank}] decode verified bit-exact on all {len(specs)} tensors")

    # inputs that fit in L2 (the small weight sets) get an L2 flush before every
    # step, outside the timed events; the 8B-shaped set touches 26.7 GB per step
    flush = None
    if read_bytes + 2 * n_total <= L2_FLUSH_BELOW:
        flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    clocks = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    if flush is None:
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
        evs[0].record(stream)
        for k in range(args.steps):
            dec.run(err, stream)
            evs[k + 1].record(stream)
        torch.cuda.synchronize()
        step_ms = [evs[k].elapsed_time(evs[k + 1]) for k in range(args.steps)]
        total_ms = evs[0].elapsed_time(evs[-1])
    else:
        pairs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                 for _ in range(args.steps)]
        for a, b in pairs:
            flush.zero_()
            a.record(stream)
            dec.run(err, stream)
            b.record(stream)
        torch.cuda.synchronize()
        step_ms = [a.elapsed_time(b) for a, b in pairs]
        total_ms = sum(step_ms)
    barrier(world)
    clk = clocks.stop()
    total_ms_max = max_over_ranks(total_ms, world, dev)
    assert api.df_read_error(err) == 0
    ms_per_step = total_ms_max / args.steps
    bf16_bytes = 2 * n_total
    value = world * bf16_bytes * args.steps / (total_ms_max / 1e3) / 1e9

    # roofline of the decode kernel (one launch per step)
    peak, peak_src = measured_hbm_peak()
    algo_bytes = read_bytes + bf16_bytes
    enc_algo = 2 * bf16_bytes + n_total + sum(c.sizes["stream_bytes"] for c in comps)
    launch_ms = statistics.mean(step_ms)
    achieved = algo_bytes / (launch_ms / 1e3) / 1e9
    traffic = None
    rec = decode_traffic_record()
    if rec and args.workload == "llama8b_shaped":
        traffic = int(rec["dram_bytes_per_weight"] * n_total)

    # ---- (ii) layer by layer into one reused buffer: the tensors of one decoder
    # layer share a buffer; every other tensor (embedding, lm_head, ...) uses a
    # second one
    groups = []
    for i, s in enumerate(specs):
        parts = s.name.split(".")
        key = ".".join(parts[:2]) if parts[0] == "layers" else None
        if key is not None and groups and groups[-1][0] == key:
            groups[-1][1].append(i)
        else:
            groups.append((key, [i]))
    layer_need = max([sum(specs[j].numel for j in idx) for key, idx in groups if key] or [0])
    other_need = max([specs[idx[0]].numel for key, idx in groups if not key] or [0])
    layer_buf = torch.empty(layer_need, dtype=torch.int16, device=dev) if layer_need else None
    other_buf = torch.empty(other_need, dtype=torch.int16, device=dev) if other_need else None
    layer_groups = []
    for key, idx in groups:
        buf = layer_buf if key else other_buf
        views, off = [], 0
        for j in idx:
            views.append(buf[off: off + specs[j].numel])
            off += specs[j].numel
        layer_groups.append((idx, views))
    layer_decs = [codec.BatchDecoder([comps[j] for j in idx], views) for idx, views in layer_groups]
    for (idx, views), d in zip(layer_groups, layer_decs):  # verify each group once
        d.run(err)
        for j, v in zip(idx, views):
            if not torch.equal(v, src[j]):
                raise SystemExit(f"layer-by-layer decode mismatch on {specs[j].name}")
    lsteps = max(1, args.steps // 4)
    for _ in range(args.warmup):
        for d in layer_decs:
            d.run(err)
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(lsteps):
        for d in layer_decs:
            d.run(err, stream)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    lbl_ms = max_over_ranks(e0.elapsed_time(e1), world, dev) / lsteps
    assert api.df_read_error(err) == 0

    # ---- e2e through the public API: pinned host container -> device -> decode -> pinned host BF16
    host_parts = []
    for c in comps:
        host_parts.append({k: getattr(c, k).cpu().pin_memory() for k in ("stream", "gaps", "offsets")} |
                          {"sm": c.sm[: c.n].cpu().pin_memory()})
    host_out = torch.empty(max(sum(comps[j].n for j in idx) for idx, _ in layer_groups), dtype=torch.int16,
                           pin_memory=True)
    h2d = sum(sum(p.numel() * p.element_size() for p in hp.values()) for hp in host_parts)
    d2h = bf16_bytes

    def e2e_step():
        for (idx, views), d in zip(layer_groups, layer_decs):
            for j in idx:
                c, hp = comps[j], host_parts[j]
                c.stream.copy_(hp["stream"], non_blocking=True)
                c.gaps.copy_(hp["gaps"], non_blocking=True)
                c.offsets.copy_(hp["offsets"], non_blocking=True)
                c.sm[: c.n].copy_(hp["sm"], non_blocking=True)
            d.run(err)
            off = 0
            for v in views:
                host_out[off: off + v.numel()].copy_(v, non_blocking=True)
                off += v.numel()

    e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    t0 = time.perf_counter()
    e0.record(stream)
    for _ in range(args.e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    wall = time.perf_counter() - t0
    barrier(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev) / args.e2e_steps
    assert api.df_read_error(err) == 0
    # the last decoded group is still in host_out: check it against the source
    idx, views = layer_groups[-1]
    off = 0
    for j in idx:
        if not torch.equal(host_out[off: off + comps[j].n], src[j].cpu()):
            raise SystemExit("e2e output mismatch")
        off += comps[j].n

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_sample(specs)

    if rank == 0:
        line = {
            "metric": METRIC,
            "value": round(value, 2),
            "unit": "GB/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": round(ms_per_step, 4),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "u8",
            "data": "synthetic (seeded; Box-Muller normals rounded to BF16, shapes of an 8B Llama-style model)",
            "config": {"workload": WORKLOAD if args.workload == "llama8b_shaped" else args.workload,
                       "weights": n_total, "tensors": len(specs),
                       "chunk_bytes": args.chunk_bytes or "32 (16 for tensors whose shortest code is 1 bit)",
                       "threads_per_block": args.threads_per_block, "max_len": 32,
                       "l2": f"inputs ({(read_bytes + bf16_bytes) / 1e9:.2f} GB) larger than L2: no flush"
                       if flush is None else
                       f"L2 flushed before every step ({L2_FLUSH_BYTES >> 20} MiB written, outside the timed "
                       f"events)",
                       "parallelism": f"{world} replica(s), no collective" if world > 1 else "1 GPU"},
            "weights_per_s": round(world * n_total * args.steps / (total_ms_max / 1e3), 1),
            "compressed_pct": round(100.0 * container / bf16_bytes, 4),
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(achieved / peak, 4), "traffic": traffic,
                         "peak_source": peak_src,
                         "kernel": "decode_kernel<BatchSrc> (df_decode_batch_run), one launch per step",
                         "algorithmic_bytes_per_launch": algo_bytes},
            "step_ms": {"median": round(statistics.median(step_ms), 4), "min": round(min(step_ms), 4),
                        "max": round(max(step_ms), 4)},
            "layer_by_layer": {"value": round(world * bf16_bytes / (lbl_ms / 1e3) / 1e9, 2), "unit": "GB/s",
                               "ms_per_pass": round(lbl_ms, 4), "launches_per_pass": len(layer_decs),
                               "steps": lsteps},
            "encode": {"value": round(bf16_bytes / ((hist_ms + enc_ms) / 1e3) / 1e9, 2), "unit": "GB/s of BF16 input",
                       "histogram_ms": round(hist_ms, 3), "encode_ms": round(enc_ms, 3),
                       "roofline_frac": round(enc_algo / ((hist_ms + enc_ms) / 1e3) / 1e9 / peak, 4),
                       "algorithmic_bytes": enc_algo,
                       "note": "device time of df_histogram over all tensors back to back, plus df_encode over "
                               "all tensors back to back (the host code build between them is not timed); "
                               "algorithmic bytes: the input read twice (histogram, pack) + sign|fraction "
                               "bytes + stream written"},
            "e2e": {"value": round(world * bf16_bytes / (e2e_ms / 1e3) / 1e9, 3), "unit": "GB/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 2),
                    "wall_s": round(wall / args.e2e_steps, 3),
                    "how": "per layer: pinned host container parts -> HBM (cudaMemcpyAsync via torch), "
                           "df_decode_batch_run, BF16 -> pinned host buffer; one stream"},
            "gpu_launches": args.steps,
            "clocks": clk,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)


def main():
    args = parse()
    world, rank, local = dist_setup()
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_gpu(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
