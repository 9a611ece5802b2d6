"""Benchmark: BF16 decode GB/s of the 8B-shaped weight set on B200, with the
fraction of the HBM roofline and the compressed size as % of BF16.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one full decode of the llama8b_shaped weight set (32 decoder layers
of q/o 4096x4096, k/v 1024x4096, gate/up 14336x4096, down 4096x14336 and two
4096 norms, plus a 128256x4096 embedding and lm_head: 8,030,257,152 BF16
weights, 16.06 GB) by ONE grouped launch (df_decode_batch_run) from the
compressed containers resident in HBM into 16.06 GB of BF16 outputs. The inputs
are far larger than L2, so no L2 flush is needed between steps.

Also reported on the same line (N = 1 unless said otherwise):
  configs         decode GB/s, weights/s, roofline fraction and compressed % of
                  every weight set (single_1024x4096, llama_layer,
                  heavy_tail_64m, llama8b_shaped, mixed_2000); sets that fit in
                  L2 get an L2 flush before every timed step. Each set also
                  carries "nf12": the same figures for the fixed 12-bit format
                  on the same tensors, with its encoder's device time; the
                  main set also carries "idx8": its containers with the
                  compact block index in place of the uint64 offsets
  layer_by_layer  the 8B-shaped set decoded layer by layer into reused buffers
  jit_layer       per-step overhead of decoding each layer just in time, one or
                  two layers ahead of a GEMM consumer, against BF16-resident
                  weights
  encode          device time of the GPU encoder, per call summed
  e2e             through the public API from pinned host memory: containers
                  copied in and BF16 copied out every step, overlapped with the
                  decode layer by layer (every N); into_hbm: the same with the
                  BF16 left in HBM for an on-GPU consumer
  verify          device SHA-256 (leaf tree) and compare throughput on the
                  decoded set
  roofline        the decode kernel against the measured HBM copy bandwidth
  cpu_baseline    the oracle on the host cores, on a bounded sample
  clocks          SM clocks sampled during the timed region

With N > 1 (torchrun), the tensors are partitioned over the ranks (balanced
by the bytes each decode moves; no data-path collective, since tensors decode
independently): every rank decodes its own share from its own HBM, `value` =
all ranks' BF16 bytes over the slowest rank's time (strong scaling).

--impl reference times the CPU oracle (the plain single-threaded decoder) on
the host cores on a bounded sample of the same workload, same metric and unit.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import platform
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
NOMINAL_HBM_GBS = 8000.0
SMALL_SETS = ("single_1024x4096", "heavy_tail_64m", "mixed_2000")


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--e2e-steps", type=int, default=2)
    p.add_argument("--workload", default="llama8b_shaped",
                   choices=["llama8b_shaped", "llama_layer", "single_1024x4096", "heavy_tail_64m", "mixed_2000"],
                   help="weight set of the headline number (llama8b_shaped by default)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-extras", action="store_true",
                   help="headline only: skip the per-set records, layer-by-layer and jit_layer")
    p.add_argument("--jit-tokens", default="4096,16384",
                   help="activation rows of the jit_layer GEMM consumer (comma-separated sizes)")
    p.add_argument("--jit-layers", type=int, default=32, help="decoder layers in the jit_layer measurement")
    p.add_argument("--chunk-bytes", type=int, default=0,
                   help="format chunk size C in bytes (0: 32, or 16 where the shortest code is 1 bit)")
    p.add_argument("--threads-per-block", type=int, default=32, help="format block size T in chunks")
    return p.parse_args()


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        backend = "nccl" if _cuda_ok() else "gloo"
        if backend == "nccl":
            import torch

            torch.cuda.set_device(local)  # NCCL binds each rank's communicator to its own GPU
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=600))
    return world, rank, local


def _cuda_ok():
    import torch

    return torch.cuda.is_available()


def _reduce(x: float, world: int, device, op: str) -> float:
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
    return float(t.item())


def max_over_ranks(x: float, world: int, device=None) -> float:
    return _reduce(x, world, device, "max")


def sum_over_ranks(x: float, world: int, device=None) -> float:
    return _reduce(x, world, device, "sum")


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


def decode_traffic_record(workload: str):
    """ncu DRAM bytes of one decode launch captured on `workload` with the
    current kernel source (profiles/decode_traffic.json), or None."""
    path = os.path.join(ROOT, "profiles", "decode_traffic.json")
    src = os.path.join(ROOT, "lossless_bf16_weight_huffman_b200", "csrc", "df_decode.cu")
    try:
        caps = json.load(open(path))["captures"]
    except Exception:
        return None
    digest = source_digest([src])
    for rec in caps:
        if rec.get("workload") == workload and rec.get("kernel_source_sha") == digest:
            return rec
    return None


# ---------------------------------------------------------------------------------------------
# the oracle on the host cores (reference arm and cpu_baseline); test infrastructure, never on
# the GPU path


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
        "scaling": "strong", "vs_baseline": None, "dtype": "u8", "data": "synthetic", "impl": "reference",
        "config": {"workload": WORKLOAD, "sample": "layers.0.q_proj (16,777,216 weights) per step",
                   "parallelism": "host, single thread"},
        "compressed_pct": round(100.0 * enc.container_bytes / (2 * w.size), 3),
        "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": "layers.0.q_proj decoded bit-serially, 16,777,216 weights per step"},
        "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def _oracle_job(job):
    """One tensor through the oracle in a worker process: (weights, encode s, decode s)."""
    set_name, index = job
    import oracle
    from lossless_bf16_weight_huffman_b200 import synth

    w = synth.generate(synth.weight_set(set_name)[index])
    t0 = time.perf_counter()
    enc = oracle.encode(w)
    t1 = time.perf_counter()
    out = oracle.decode_encoded(enc)
    t2 = time.perf_counter()
    if not (out == w).all():
        raise RuntimeError(f"oracle round trip failed on {set_name}[{index}]")
    return int(w.size), t1 - t0, t2 - t1


def _nf12_oracle_job(job):
    """One tensor through the fixed 12-bit format's oracle: (weights, encode s, decode s)."""
    set_name, index = job
    from lossless_bf16_weight_huffman_b200 import synth
    from oracle import nf12_oracle

    w = synth.generate(synth.weight_set(set_name)[index])
    t0 = time.perf_counter()
    slots, bitmap, side = nf12_oracle.encode(w)
    t1 = time.perf_counter()
    back = nf12_oracle.decode(slots, bitmap, side, w.size)
    t2 = time.perf_counter()
    if not (back == w).all():
        raise RuntimeError(f"nf12 oracle round trip failed on {set_name}[{index}]")
    return int(w.size), t1 - t0, t2 - t1


def _cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return platform.processor() or "unknown"


def cpu_baseline(pool, ncores):
    """The oracle encoder and decoder on bounded samples of every weight set,
    one process (one host thread) per tensor across all host cores; a
    worker's own times give the one-thread rates. The fixed 12-bit format's
    oracle (numpy) runs on the same tensors in the same workers. The 8B-shaped set is
    extrapolated from a decoder layer (same shapes and distributions) by
    weight count."""
    from lossless_bf16_weight_huffman_b200 import synth

    samples = {
        "single_1024x4096": [("single_1024x4096", 0)],
        "llama_layer": [("llama_layer", i) for i in range(len(synth.llama_layer()))],
        "heavy_tail_64m": [("heavy_tail_64m", 0)],
        "mixed_2000": [("mixed_2000", i) for i in range(0, 2000, 8)],  # every 8th tensor
    }
    per = {}
    for name, jobs in samples.items():
        t0 = time.perf_counter()
        multi = pool.map(_oracle_job, jobs)
        wall = time.perf_counter() - t0
        n = sum(m[0] for m in multi)
        rec = {"weights": n, "all_cores_wall_s": round(wall, 3),
               "all_cores_gbs_roundtrip": round(2 * n / wall / 1e9, 4)}
        # every worker is one host thread: the sum of its times is the
        # one-thread time
        enc_s = sum(m[1] for m in multi)
        dec_s = sum(m[2] for m in multi)
        rec.update({"one_thread_encode_gbs": round(2 * n / enc_s / 1e9, 4),
                    "one_thread_decode_gbs": round(2 * n / dec_s / 1e9, 4),
                    "one_thread_weights_per_s": round(n / dec_s, 1)})
        nf = pool.map(_nf12_oracle_job, jobs)  # after the timed pass: its wall time is the Huffman oracle's
        rec.update({"nf12_one_thread_encode_gbs": round(2 * n / max(sum(m[1] for m in nf), 1e-9) / 1e9, 4),
                    "nf12_one_thread_decode_gbs": round(2 * n / max(sum(m[2] for m in nf), 1e-9) / 1e9, 4)})
        if name == "mixed_2000":
            rec["sample"] = "every 8th tensor (250 of 2000)"
        per[name] = rec
    layer = per["llama_layer"]
    return {
        "value": layer["one_thread_decode_gbs"], "unit": "GB/s", "cores": 1, "kind": "oracle",
        "sample": "decoder layer (218,112,000 weights of the 8B shapes), bit-serial decode, one host thread; "
                  "8B-shaped set extrapolated by weight count",
        "host": {"nproc": ncores, "cpu_model": _cpu_model()},
        "all_cores": {"value": layer["all_cores_gbs_roundtrip"], "unit": "GB/s (encode + decode round trip)",
                      "cores": min(ncores, len(synth.llama_layer())),
                      "how": "one process per tensor (spawned before the first GPU call)"},
        "per_set": per,
    }


# ---------------------------------------------------------------------------------------------
# GPU side


def encode_set(specs, dev, args, staging):
    """Generate each tensor on the host, copy it to HBM and encode it there.
    Returns (source tensors, containers, histogram device ms, encode device ms).
    All df_histogram calls are captured in one CUDA graph and all df_encode
    calls in another; each graph is replayed once to produce the results and
    once more under CUDA events, so the times are device time without host
    launch gaps."""
    import numpy as np
    import torch

    from lossless_bf16_weight_huffman_b200 import api, codec, synth

    src = []
    for s in specs:
        n = s.numel
        synth.fill_ptr(s, staging.data_ptr(), n)
        x = torch.empty(n, dtype=torch.int16, device=dev)
        x.copy_(staging[:n])
        torch.cuda.synchronize()  # the staging buffer is refilled next
        src.append(x)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    hist_d = torch.empty((len(specs), 256), dtype=torch.int64, device=dev)

    def graph_of(calls):
        side = torch.cuda.Stream(dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(side), torch.cuda.graph(g, stream=side):
            calls()
        torch.cuda.synchronize(dev)
        return g

    def replay_ms(g):
        g.replay()  # the results
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        g.replay()
        b.record()
        torch.cuda.synchronize(dev)
        return a.elapsed_time(b)

    g_hist = graph_of(lambda: [api.df_histogram(x, hist_d[i]) for i, x in enumerate(src)])
    hist_ms = replay_ms(g_hist)
    hists = hist_d.cpu().numpy().view(np.uint64)
    plans = []
    for i, s in enumerate(specs):
        code = api.df_build_code(hists[i], 32)
        C = args.chunk_bytes or codec.auto_chunk_bytes(code)
        T = args.threads_per_block
        lut = torch.from_numpy(api.df_build_lut(code).view(np.int32)).to(dev)
        z = api.df_plan(code, hists[i], s.numel, C, T).as_dict()
        bufs = dict(stream=torch.empty(z["stream_bytes"], dtype=torch.uint8, device=dev),
                    gaps=torch.empty(z["gap_bytes"], dtype=torch.uint8, device=dev),
                    offsets=torch.empty(z["n_blocks"] + 1, dtype=torch.int64, device=dev),
                    sm=torch.empty(max(s.numel, 16), dtype=torch.uint8, device=dev))
        plans.append((code, C, T, lut, z, bufs))
    ws = torch.empty(max(p[4]["encode_ws_bytes"] for p in plans), dtype=torch.uint8, device=dev)
    torch.cuda.synchronize()

    def encodes():
        for x, (code, C, T, lut, z, bufs) in zip(src, plans):
            api.df_encode(code, x, z["total_bits"], C, T, bufs["stream"], bufs["gaps"], bufs["offsets"],
                          bufs["sm"], ws, err)

    enc_ms = replay_ms(graph_of(encodes))
    assert api.df_read_error(err) == 0, "encode reported an error"
    comps = [codec.Compressed(n=s.numel, shape=s.shape, code=code, lut=lut, sizes=z, chunk_bytes=C,
                              threads_per_block=T, **bufs)
             for s, (code, C, T, lut, z, bufs) in zip(specs, plans)]
    return src, comps, hist_ms, enc_ms


def grouped_encode_record(src, comps, args, peak, steps=5):
    """The grouped encoder (codec.BatchEncoder: one histogram launch, then one
    zeroing launch and one encode launch for all tensors) on the same tensors:
    its containers against those of the per-tensor calls, and its device time
    per step (CUDA events around each part, median of `steps`; inputs not
    flushed from L2 between steps)."""
    import statistics

    import torch

    from lossless_bf16_weight_huffman_b200 import api, codec

    n = sum(x.numel() for x in src)
    enc = codec.BatchEncoder(src, chunk_bytes=args.chunk_bytes, threads_per_block=args.threads_per_block)
    got = enc.prepare()
    err = torch.zeros(1, dtype=torch.int32, device=src[0].device)
    enc.run(err)
    torch.cuda.synchronize()
    flags = api.df_read_error(err)
    equal = flags == 0 and all(
        a.total_bits == b.total_bits and torch.equal(a.stream, b.stream) and torch.equal(a.gaps, b.gaps)
        and torch.equal(a.offsets, b.offsets) and torch.equal(a.sm[: a.n], b.sm[: b.n])
        for a, b in zip(got, comps))
    hist_t, enc_t = [], []
    for _ in range(steps):
        e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        e0.record()
        enc.run_histograms()
        e1.record()
        enc.run(err)
        e2.record()
        torch.cuda.synchronize()
        hist_t.append(e0.elapsed_time(e1))
        enc_t.append(e1.elapsed_time(e2))
    h, e = statistics.median(hist_t), statistics.median(enc_t)
    algo = 4 * n + n + sum(c.sizes["stream_bytes"] for c in comps)
    del enc, got
    torch.cuda.empty_cache()
    return {"value": round(2 * n / ((h + e) / 1e3) / 1e9, 2), "unit": "GB/s of BF16 input",
            "histogram_ms": round(h, 4), "encode_ms": round(e, 4),
            "roofline_frac": round(algo / ((h + e) / 1e3) / 1e9 / peak, 4),
            "equal_to_per_tensor_calls": bool(equal), "error_flags": flags, "tensors": len(src),
            "note": "df_histogram_batch_run (a memset, one kernel) and df_encode_batch_run (a zeroing kernel, a "
                    "memset, one encode kernel) over all tensors; algorithmic bytes as the per-tensor record"}


def recorded(fn, *args):
    """fn(*args), or the exception it raised as the record (so that one
    secondary measurement cannot cost the whole bench line)."""
    try:
        return fn(*args)
    except Exception as e:  # reported in the JSON line, not hidden
        return {"error": f"{type(e).__name__}: {e}"}


def time_launches(run, steps, warmup, stream, flush=None):
    """Per-step device ms of run() (CUDA events on `stream`). With `flush`, a
    write larger than L2 precedes every step, outside its events."""
    import torch

    for _ in range(max(warmup, 1)):
        run()
    torch.cuda.synchronize()
    if flush is None:
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
        evs[0].record(stream)
        for k in range(steps):
            run()
            evs[k + 1].record(stream)
        torch.cuda.synchronize()
        return [evs[k].elapsed_time(evs[k + 1]) for k in range(steps)]
    pairs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for a, b in pairs:
        flush.zero_()
        a.record(stream)
        run()
        b.record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in pairs]


def verify(src, outs, names):
    import torch

    for x, o, name in zip(src, outs, names):
        if not torch.equal(x, o.view(torch.int16).reshape(-1)):
            raise SystemExit(f"decode mismatch on {name}")


def decode_record(comps, outs, args, stream, err, peak, flush):
    """Decode timing of one grouped launch over `comps`: GB/s of BF16 out,
    weights/s, roofline fraction of the algorithmic bytes."""
    from lossless_bf16_weight_huffman_b200 import api, codec

    dec = codec.BatchDecoder(comps, outs)
    n = sum(c.n for c in comps)
    read = sum(c.read_bytes() for c in comps)
    use_flush = flush is not None and read + 2 * n <= L2_FLUSH_BELOW
    ms = time_launches(lambda: dec.run(err, stream), args.steps, args.warmup, stream, flush if use_flush else None)
    assert api.df_read_error(err) == 0
    med = statistics.median(ms)
    algo = read + 2 * n
    return {"gbs": round(2 * n / med / 1e6, 2), "weights_per_s": round(n / med * 1e3, 1),
            "ms": round(med, 4), "roofline_frac": round(algo / med / 1e6 / peak, 4),
            "compressed_pct": round(100.0 * sum(c.container_bytes for c in comps) / (2 * n), 4),
            "weights": n, "tensors": len(comps),
            "l2": "flushed before every step" if use_flush else "inputs larger than L2: no flush"}


def nf12_record(src, outs, args, stream, err, peak, flush):
    """The fixed 12-bit format on the same tensors: compressed size, one
    grouped decode launch per step (GB/s, weights/s, roofline fraction of its
    algorithmic bytes), and the grouped encoder's device time (its launches
    captured as one CUDA graph, replayed under CUDA events)."""
    import torch

    from lossless_bf16_weight_huffman_b200 import api, nf12

    encoder = nf12.BatchEncoder(src)
    comps = encoder.run(err)
    dec = nf12.BatchDecoder(comps, outs)
    n = sum(c.n for c in comps)
    read = sum(c.read_bytes() for c in comps)
    use_flush = flush is not None and read + 2 * n <= L2_FLUSH_BELOW
    ms = time_launches(lambda: dec.run(err, stream), args.steps, args.warmup, stream, flush if use_flush else None)
    assert api.df_read_error(err) == 0
    verify(src, outs, [f"nf12 tensor {i}" for i in range(len(src))])
    med = statistics.median(ms)
    dev = src[0].device
    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side), torch.cuda.graph(g, stream=side):
        api.df_nf12_encode_batch_groups(encoder.plan, encoder.escaped)
        api.df_nf12_encode_batch_escapes(encoder.plan, err)
    torch.cuda.synchronize(dev)
    g.replay()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    g.replay()
    b.record()
    torch.cuda.synchronize(dev)
    enc_ms = a.elapsed_time(b)
    assert api.df_read_error(err) == 0
    del g
    enc_bytes = sum(2 * c.n + 12 * c.groups + 4 * ((c.groups + 31) // 32) + 32 * c.n_escaped for c in comps)
    return {"compressed_pct": round(100.0 * sum(c.container_bytes for c in comps) / (2 * n), 4),
            "escaped_groups_pct": round(100.0 * sum(c.n_escaped for c in comps) / max(1, sum(c.groups for c in comps)), 4),
            "gbs": round(2 * n / med / 1e6, 2), "weights_per_s": round(n / med * 1e3, 1), "ms": round(med, 4),
            "roofline_frac": round((read + 2 * n) / med / 1e6 / peak, 4),
            "encode_ms": round(enc_ms, 4),
            "encode_roofline_frac": round(enc_bytes / enc_ms / 1e6 / peak, 4),
            "l2": "flushed before every step" if use_flush else "inputs larger than L2: no flush"}


def idx8_record(comps, outs, src, args, stream, err, peak, flush):
    """The same containers with the compact block index in place of the
    uint64 offsets: index bytes, the index build's device time (all builds
    as one CUDA graph), and one grouped decode launch per step through it."""
    import torch

    from lossless_bf16_weight_huffman_b200 import api, codec

    ix = [codec.Compressed(n=c.n, shape=c.shape, code=c.code, lut=c.lut, sizes=c.sizes, chunk_bytes=c.chunk_bytes,
                           threads_per_block=c.threads_per_block, stream=c.stream, gaps=c.gaps, offsets=c.offsets,
                           sm=c.sm).use_index8() for c in comps]
    dev = comps[0].stream.device
    wide = torch.zeros(1, dtype=torch.int64, device=dev)
    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side), torch.cuda.graph(g, stream=side):
        for c, d in zip(comps, ix):
            api.df_index8_build(c.offsets, c.sizes["n_blocks"], d.index8, wide, err)
    torch.cuda.synchronize(dev)
    g.replay()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    g.replay()
    b.record()
    torch.cuda.synchronize(dev)
    build_ms = a.elapsed_time(b)
    del g
    rec = decode_record(ix, outs, args, stream, err, peak, flush)
    verify(src, outs, [f"tensor {i} through the compact index" for i in range(len(src))])
    rec.update({"index_bytes": sum(c.index_bytes for c in ix),
                "u64_offsets_bytes": sum(c.sizes["offsets_bytes"] for c in comps),
                "wide_superblocks": sum(c.index8_wide for c in ix),
                "superblocks": sum((c.sizes["n_blocks"] + 63) // 64 for c in ix),
                "build_ms": round(build_ms, 4)})
    return rec


def verify_record(outs, dev):
    """Device throughput of the verify steps on the decoded set: the per-tensor
    SHA-256 leaf tree (df_sha256_device, leaf digests to the host) and the
    first-difference compare (df_compare) of every output with itself."""
    import torch

    from lossless_bf16_weight_huffman_b200 import api

    nbytes = sum(2 * o.numel() for o in outs)
    ws = torch.empty(max(api.df_sha256_workspace(2 * o.numel()) for o in outs), dtype=torch.uint8, device=dev)
    first = torch.empty(1, dtype=torch.int64, device=dev)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for o in outs:
        api.df_sha256_device(o, ws)  # waits for its leaf digests
    t_sha = time.perf_counter() - t0
    big = max(outs, key=lambda o: o.numel())
    api.df_sha256_device(big, ws)
    t0 = time.perf_counter()
    api.df_sha256_device(big, ws)
    t_big = time.perf_counter() - t0
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for o in outs:
        api.df_compare(o, o, first)
    b.record()
    torch.cuda.synchronize()
    t_cmp = a.elapsed_time(b) / 1e3
    return {"sha256_gbs": round(nbytes / t_sha / 1e9, 2), "sha256_s": round(t_sha, 3),
            "sha256_largest_tensor_gbs": round(2 * big.numel() / t_big / 1e9, 2),
            "compare_gbs": round(2 * nbytes / t_cmp / 1e9, 1), "bytes": nbytes,
            "note": "sha256: wall time over all tensors (290 calls, each waiting for its leaf digests and "
                    "hashing them on the host), and for the largest tensor alone; compare: device time, both "
                    "operands read"}


def layer_groups(specs, idx):
    """Indices (into idx) grouped by decoder layer; every other tensor alone."""
    groups = []
    for j, i in enumerate(idx):
        parts = specs[i].name.split(".")
        key = ".".join(parts[:2]) if parts[0] == "layers" else None
        if key is not None and groups and groups[-1][0] == key:
            groups[-1][1].append(j)
        else:
            groups.append((key, [j]))
    return groups


def jit_record(args, specs, idx, comps, outs, src, err, dev):
    """Per-pass time of a GEMM consumer over the decoder layers with weights
    (a) resident as BF16, (b) decoded just in time at run-ahead depth 0, 1, 2,
    (c) the same from the fixed 12-bit format; for every consumer size in
    --jit-tokens (the overhead is the decode time over the GEMM time, so it
    shrinks as the consumer grows)."""
    import torch

    from lossless_bf16_weight_huffman_b200 import jit, nf12

    groups = [(k, g) for k, g in layer_groups(specs, idx) if k is not None][: args.jit_layers]
    if not groups:
        return None
    layer_specs = [[specs[idx[j]] for j in g] for _, g in groups]
    ins = sorted({s.shape[1] for l in layer_specs for s in l if len(s.shape) == 2})
    outs_f = sorted({s.shape[0] for l in layer_specs for s in l if len(s.shape) == 2})
    resident = [[outs[j] for j in g] for _, g in groups]
    layers = [[comps[j] for j in g] for _, g in groups]
    n12 = [[nf12.compress(src[j]) for j in g] for _, g in groups]

    def timed(fn, reps=3):
        fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(reps):
            fn()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / reps

    def one_size(B):
        gen = torch.Generator(device=dev).manual_seed(0xDF11)
        x_in = {k: torch.randn(B, k, generator=gen, device=dev, dtype=torch.float32).to(torch.bfloat16) for k in ins}
        y_out = {k: torch.empty(B, k, device=dev, dtype=torch.bfloat16) for k in outs_f}
        flops = sum(2 * B * s.numel for l in layer_specs for s in l if len(s.shape) == 2)

        def consume(l, views):
            for s, v in zip(layer_specs[l], views):
                if len(s.shape) != 2:
                    continue
                w = v.view(torch.bfloat16).view(s.shape[0], s.shape[1])
                torch.matmul(x_in[s.shape[1]], w.t(), out=y_out[s.shape[0]])

        t_res = timed(lambda: [consume(l, resident[l]) for l in range(len(groups))])
        rec = {"consumer": f"per layer, y = x W^T for each linear weight (cuBLAS bf16), x: {B} rows",
               "layers": len(groups), "tokens": B, "gemm_tflops_resident": round(flops / t_res / 1e9, 1),
               "resident_ms_per_pass": round(t_res, 3)}
        for fmt, ls in (("", layers), ("nf12_", n12)):
            for depth in (0, 1, 2):
                st = jit.LayerStreamer(ls, depth=depth, device=dev)
                t = timed(lambda: st.run(consume))
                assert st.errors() == 0
                rec[f"{fmt}depth{depth}_ms_per_pass"] = round(t, 3)
                rec[f"{fmt}depth{depth}_overhead_pct"] = round(100.0 * (t - t_res) / t_res, 2)
                del st
        return rec

    sizes = [int(b) for b in str(args.jit_tokens).split(",") if b]
    recs = [one_size(B) for B in sizes]
    rec = dict(recs[0])
    if len(recs) > 1:
        rec["more_tokens"] = recs[1:]
    # the decode alone, layer by layer, for scale
    for fmt, ls in (("", layers), ("nf12_", n12)):
        st = jit.LayerStreamer(ls, depth=0, device=dev)
        rec[f"{fmt}decode_alone_ms_per_pass"] = round(timed(lambda: st.run(lambda l, v: None)), 3)
        del st

    # every just-in-time layer equals the resident weights (depth 1, both formats)
    def check(l, views):
        for a, b in zip(views, resident[l]):
            if not torch.equal(a, b.view(torch.int16).reshape(-1)):
                raise SystemExit(f"just-in-time decode differs from the resident weights, layer {l}")

    for ls in (layers, n12):
        st = jit.LayerStreamer(ls, depth=1, device=dev)
        st.run(check)
        torch.cuda.synchronize()
        del st
    del n12
    return rec


def e2e_record(args, specs, idx, comps, src, dev, world):
    """Through the public API from pinned host memory: per layer, the container
    parts are copied in on a copy stream, decoded on a decode stream and the
    BF16 copied back out to pinned host buffers on the consumer's stream; the
    three overlap across layers (jit.HostLayerStreamer)."""
    import torch

    from lossless_bf16_weight_huffman_b200 import jit

    groups = layer_groups(specs, idx)
    layers = [[comps[j] for j in g] for _, g in groups]
    hls = jit.HostLayerStreamer(layers, device=dev)
    cap = max(sum(c.n for c in l) for l in layers)
    host_out = [torch.empty(cap, dtype=torch.int16, pin_memory=True) for _ in range(2)]

    def consume(i, views):
        off, dst = 0, host_out[i % 2]
        for v in views:
            dst[off: off + v.numel()].copy_(v, non_blocking=True)
            off += v.numel()

    hls.run(consume)
    torch.cuda.synchronize()
    assert hls.errors() == 0
    # the same stream into HBM only (the consumer keeps the BF16 on the GPU;
    # the step's result read back is the decode status word)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    hls.run(lambda i, views: None)
    torch.cuda.synchronize()
    a.record()
    for _ in range(args.e2e_steps):
        hls.run(lambda i, views: None)
        assert hls.errors() == 0  # reads the status word back each step
    b.record()
    torch.cuda.synchronize()
    ms_in = max_over_ranks(a.elapsed_time(b) / args.e2e_steps, world, dev)
    last = groups[-1][1]
    off = 0
    for j in last:
        if not torch.equal(host_out[(len(groups) - 1) % 2][off: off + comps[j].n], src[j].cpu()):
            raise SystemExit("e2e output mismatch")
        off += comps[j].n
    barrier(world)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0 = time.perf_counter()
    a.record()
    for _ in range(args.e2e_steps):
        hls.run(consume)
    b.record()
    torch.cuda.synchronize()
    wall = (time.perf_counter() - t0) / args.e2e_steps
    ms = max_over_ranks(a.elapsed_time(b) / args.e2e_steps, world, dev)
    n_all = sum_over_ranks(sum(c.n for c in comps), world, dev)
    return {"value": round(2 * n_all / (ms / 1e3) / 1e9, 3), "unit": "GB/s",
            "h2d_bytes_per_step": int(sum_over_ranks(hls.h2d_bytes, world, dev)),
            "d2h_bytes_per_step": int(2 * n_all), "ms_per_step": round(ms, 2), "wall_s": round(wall, 3),
            "how": "jit.HostLayerStreamer: per layer, pinned host container -> HBM on a copy stream, "
                   "df_decode_batch_run on a decode stream, BF16 -> pinned host on the consumer stream; "
                   "consecutive layers overlap",
            "into_hbm": {"value": round(2 * n_all / (ms_in / 1e3) / 1e9, 3), "unit": "GB/s of BF16 decoded",
                         "ms_per_step": round(ms_in, 2), "d2h_bytes_per_step": 4 * world,
                         "how": "the same, the BF16 left in HBM for an on-GPU consumer; the decode status "
                                "word read back every step"}}


def run_gpu(args, world, rank, local, pool, ncores):
    import torch

    from lossless_bf16_weight_huffman_b200 import build, codec, shard, synth

    build.build_all()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    peak, peak_src = measured_hbm_peak()
    all_specs = synth.weight_set(args.workload)
    parts = shard.partition([s.numel for s in all_specs], world)
    idx = parts[rank]
    specs = [all_specs[i] for i in idx]
    n_all = sum(s.numel for s in all_specs)
    n_mine = sum(s.numel for s in specs)

    # ---- this rank's share: generated on the host, encoded on the GPU
    t_setup = time.time()
    staging = torch.empty(max([s.numel for s in specs] + [1]), dtype=torch.int16, pin_memory=True)
    src, comps, hist_ms, enc_ms = encode_set(specs, dev, args, staging)
    container = sum(c.container_bytes for c in comps)
    read_bytes = sum(c.read_bytes() for c in comps)
    log(f"[rank {rank}] setup {time.time() - t_setup:.1f} s: {len(specs)} of {len(all_specs)} tensors, "
        f"{n_mine:,} weights, container {100 * container / (2 * max(n_mine, 1)):.3f}% of BF16")

    # ---- (i) the share decoded by one grouped launch per step
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    outs = [torch.empty(c.n, dtype=torch.int16, device=dev) for c in comps]
    dec = codec.BatchDecoder(comps, outs)
    dec.run(err)
    torch.cuda.synchronize()
    assert codec.api.df_read_error(err) == 0, "decode reported an error"
    verify(src, outs, [s.name for s in specs])
    log(f"[rank {rank}] decode verified bit-exact on all {len(specs)} tensors")
    flush = None
    if read_bytes + 2 * n_mine <= L2_FLUSH_BELOW:
        flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    clocks = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    step_ms = time_launches(lambda: dec.run(err, stream), args.steps, args.warmup, stream, flush)
    barrier(world)
    clk = clocks.stop()
    assert codec.api.df_read_error(err) == 0
    total_ms_max = max_over_ranks(sum(step_ms), world, dev)
    ms_per_step = total_ms_max / args.steps
    value = 2 * n_all * args.steps / (total_ms_max / 1e3) / 1e9
    container_all = sum_over_ranks(container, world, dev)
    algo_bytes = read_bytes + 2 * n_mine
    launch_ms = statistics.mean(step_ms)
    achieved = algo_bytes / (launch_ms / 1e3) / 1e9
    rec = decode_traffic_record(args.workload) if world == 1 else None
    traffic = int(rec["dram_bytes_read"] + rec["dram_bytes_write"]) if rec else None
    w_max = max_over_ranks(n_mine, world, dev)
    w_min = -max_over_ranks(-n_mine, world, dev)

    # ---- extras at N = 1
    extras = {}
    if world == 1 and not args.no_extras:
        # layer by layer into reused buffers
        groups = layer_groups(all_specs, idx)
        cap_l = max([sum(comps[j].n for j in g) for k, g in groups if k] or [0])
        cap_o = max([comps[g[0]].n for k, g in groups if not k] or [0])
        lbuf = torch.empty(max(cap_l, 1), dtype=torch.int16, device=dev)
        obuf = torch.empty(max(cap_o, 1), dtype=torch.int16, device=dev)
        decs = []
        for k, g in groups:
            buf, off, views = (lbuf if k else obuf), 0, []
            for j in g:
                views.append(buf[off: off + comps[j].n])
                off += comps[j].n
            decs.append(codec.BatchDecoder([comps[j] for j in g], views))
        lsteps = max(1, args.steps // 4)
        ms = time_launches(lambda: [d.run(err, stream) for d in decs], lsteps, args.warmup, stream)
        assert codec.api.df_read_error(err) == 0
        lbl = statistics.median(ms)
        extras["layer_by_layer"] = {"value": round(2 * n_mine / (lbl / 1e3) / 1e9, 2), "unit": "GB/s",
                                    "ms_per_pass": round(lbl, 4), "launches_per_pass": len(decs), "steps": lsteps}
        del decs, lbuf, obuf
        # every weight set: one grouped launch each
        cfg = {args.workload: {"gbs": round(2 * n_mine / launch_ms / 1e6, 2),
                               "weights_per_s": round(n_mine / launch_ms * 1e3, 1),
                               "ms": round(statistics.median(step_ms), 4),
                               "roofline_frac": round(algo_bytes / launch_ms / 1e6 / peak, 4),
                               "compressed_pct": round(100.0 * container / (2 * n_mine), 4),
                               "weights": n_mine, "tensors": len(comps),
                               "l2": "flushed before every step" if flush is not None else
                               "inputs larger than L2: no flush"}}
        fl = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
        cfg[args.workload]["nf12"] = nf12_record(src, outs, args, stream, err, peak, fl)
        torch.cuda.empty_cache()
        cfg[args.workload]["idx8"] = idx8_record(comps, outs, src, args, stream, err, peak, fl)
        extras["encode_grouped"] = recorded(grouped_encode_record, src, comps, args, peak)
        for name in ("single_1024x4096", "llama_layer", "heavy_tail_64m", "mixed_2000"):
            if name == args.workload:
                continue
            sp = synth.weight_set(name)
            stg = torch.empty(max(s.numel for s in sp), dtype=torch.int16, pin_memory=True)
            s_src, s_comps, _, _ = encode_set(sp, dev, args, stg)
            s_outs = [torch.empty(c.n, dtype=torch.int16, device=dev) for c in s_comps]
            cfg[name] = decode_record(s_comps, s_outs, args, stream, err, peak, fl)
            verify(s_src, s_outs, [s.name for s in sp])
            cfg[name]["nf12"] = nf12_record(s_src, s_outs, args, stream, err, peak, fl)
            cfg[name]["encode_grouped"] = recorded(grouped_encode_record, s_src, s_comps, args, peak)
            del s_src, s_comps, s_outs, stg
        extras["configs"] = cfg
        del fl
        if args.workload == "llama8b_shaped":
            extras["jit_layer"] = jit_record(args, all_specs, idx, comps, outs, src, err, dev)
        extras["verify"] = verify_record(outs, dev)
        torch.cuda.empty_cache()

    # ---- e2e through the public API (every N)
    e2e = e2e_record(args, all_specs, idx, comps, src, dev, world)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and pool is not None:
        cpu = cpu_baseline(pool, ncores)

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
            "scaling": "strong",
            "vs_baseline": None,
            "dtype": "u8",
            "data": "synthetic (seeded; Box-Muller normals rounded to BF16, shapes of an 8B Llama-style model)",
            "config": {"workload": WORKLOAD if args.workload == "llama8b_shaped" else args.workload,
                       "weights": n_all, "tensors": len(all_specs),
                       "chunk_bytes": args.chunk_bytes or "32 (16 for tensors whose shortest code is 1 bit)",
                       "threads_per_block": args.threads_per_block, "max_len": 32,
                       "l2": f"inputs ({(read_bytes + 2 * n_mine) / 1e9:.2f} GB per rank) larger than L2: no flush"
                       if flush is None else
                       f"L2 flushed before every step ({L2_FLUSH_BYTES >> 20} MiB written, outside the timed "
                       f"events)",
                       "parallelism": (f"{world} ranks, tensors partitioned by decode bytes (weights per rank "
                                       f"{int(w_min):,}..{int(w_max):,}), no collective")
                       if world > 1 else "1 GPU"},
            "weights_per_s": round(n_all * args.steps / (total_ms_max / 1e3), 1),
            "compressed_pct": round(100.0 * container_all / (2 * n_all), 4),
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(achieved / peak, 4), "traffic": traffic,
                         "traffic_workload": rec.get("workload") if rec else None,
                         "peak_source": peak_src,
                         "frac_of_nominal_8tbs": round(achieved / NOMINAL_HBM_GBS, 4),
                         "kernel": "decode_kernel<BatchSrc> (df_decode_batch_run), one launch per step",
                         "algorithmic_bytes_per_launch": algo_bytes},
            "step_ms": {"median": round(statistics.median(step_ms), 4), "min": round(min(step_ms), 4),
                        "max": round(max(step_ms), 4)},
            "encode": {"value": round(2 * n_mine / ((hist_ms + enc_ms) / 1e3) / 1e9, 2),
                       "unit": "GB/s of BF16 input", "histogram_ms": round(hist_ms, 3),
                       "encode_ms": round(enc_ms, 3),
                       "roofline_frac": round((4 * n_mine + n_mine + sum(c.sizes["stream_bytes"] for c in comps))
                                              / ((hist_ms + enc_ms) / 1e3) / 1e9 / peak, 4),
                       "note": "device time: all df_histogram calls replayed as one CUDA graph, then all "
                               "df_encode calls as another (CUDA events around each replay); algorithmic bytes: "
                               "the input read twice (histogram, encode pass) + sign|fraction bytes + stream "
                               "written"},
            "e2e": e2e,
            "gpu_launches": args.steps,
            "clocks": clk,
            "cpu_baseline": cpu,
        }
        line.update(extras)
        print(json.dumps(line), flush=True)


def main():
    args = parse()
    world, rank, local = dist_setup()
    pool, ncores = None, os.cpu_count() or 1
    if args.impl == "ours" and rank == 0 and world == 1 and not args.no_cpu_baseline:
        import multiprocessing as mp

        # the oracle's worker processes start before the first GPU call
        pool = mp.get_context("spawn").Pool(ncores)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_gpu(args, world, rank, local, pool, ncores)
    finally:
        if pool is not None:
            pool.close()
            pool.join()
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
