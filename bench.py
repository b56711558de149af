"""Benchmark of the split-exponent Huffman codec on one Llama-3.1-8B block.

One step = compress the block's seven BF16 weight matrices (one codebook per
matrix, one batched call) and decompress the whole block back in one batched
call (block-at-a-time, as in the DFloat11 article's "方法介绍").  `value` is
BF16 bytes encoded plus BF16 bytes decoded per second, over all ranks (each
rank codes its own block: weak scaling, no collective on the data path).

python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

--impl reference times the CPU oracle (single-threaded C++) on the host on a
bounded sample of the same workload, with the same metric.
--all-configs prints one line per workload of the codec's table (the BF16
1M and FP8 16M tensors, the block, the K/V layer, the LM head) instead.
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "exhuff decode & encode GB/s (BF16 bytes) on 218M-param block; % HBM; size ratio"
WORKLOAD = "llama8b_block"
FALLBACK_HBM_GBS = 6650.0

# DRAM traffic per decode launch on the full block, from one ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum), valid only for the decoder
# source it was taken on.
DECODE_TRAFFIC = {"bytes": 301308928 + 377901312, "source_sha": "6ceea4ebebfb7656"}


def decoder_source_sha():
    h = hashlib.sha256()
    for f in ("eh_decompress.cu", "eh_internal.cuh"):
        with open(os.path.join(ROOT, "exponent_entropy_coding_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def host_cpu_model():
    try:
        with open("/proc/cpuinfo") as fh:
            for ln in fh:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """SM clocks and throttle reasons during the timed region, polled through
    NVML about every millisecond (so that a region of a few milliseconds
    still gets several samples), else through `nvidia-smi -lms 20`.  The
    sampler is started first and the timed region begins once its first
    sample has arrived."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.samples = []  # (sm MHz, max sm MHz, set of reasons)
        self.mark = 0
        self.source = None
        self.stop = False

    def _nvml_handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        uuid = getattr(torch.cuda.get_device_properties(self.gpu), "uuid", None)
        if uuid is not None:
            u = str(uuid)
            return pynvml, pynvml.nvmlDeviceGetHandleByUUID(u if u.startswith("GPU-") else "GPU-" + u)
        return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.gpu)

    def _poll_nvml(self, nv, h):
        bits = {"hw_slowdown": nv.nvmlClocksEventReasonHwSlowdown,
                "hw_thermal_slowdown": nv.nvmlClocksEventReasonHwThermalSlowdown,
                "sw_thermal_slowdown": nv.nvmlClocksEventReasonSwThermalSlowdown,
                "sw_power_cap": nv.nvmlClocksEventReasonSwPowerCap}
        mx = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
        while not self.stop:
            try:
                sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
            except Exception:
                break
            self.samples.append((sm, mx, {k for k, v in bits.items() if r & v}))
            time.sleep(0.001)

    def _read_smi(self):
        for line in self.proc.stdout:
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm, mx = float(f[1]), float(f[2])
            except ValueError:
                continue
            self.samples.append((sm, mx, {n for n, v in zip(self.REASONS, f[5:9]) if v.lower() == "active"}))

    def __enter__(self):
        import threading
        try:
            nv, h = self._nvml_handle()
            self.thread = threading.Thread(target=self._poll_nvml, args=(nv, h), daemon=True)
            self.source = "nvml, ~1 ms"
        except Exception:
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                     "--format=csv,noheader,nounits", "-lms", "20"],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            except (OSError, ValueError):
                return self
            self.thread = threading.Thread(target=self._read_smi, daemon=True)
            self.source = "nvidia-smi, 20 ms"
        self.thread.start()
        t0 = time.time()
        while not self.samples and time.time() - t0 < 10 and self.thread.is_alive():
            time.sleep(0.001)
        self.mark = len(self.samples)  # samples from here on fall in the timed region
        return self

    def __exit__(self, *exc):
        self.stop = True
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.source:
            self.thread.join(timeout=5)
        # the sample taken just before the region started is kept as its first
        self.samples = self.samples[max(self.mark - 1, 0):]

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "source": self.source}
        reasons = set().union(*(r for _, _, r in self.samples))
        return {"sm_mhz": statistics.median(s for s, _, _ in self.samples),
                "sm_max_mhz": max(m for _, m, _ in self.samples), "reasons": sorted(reasons),
                "samples": len(self.samples), "source": self.source}


def workload_config(world, elements=218103808, chunk_elems=65536, max_code_len=32):
    """The bench line's `config`: the same for both arms."""
    return {"workload": "llama8b_block: q,k,v,o 4096/1024x4096, gate/up 14336x4096, "
                        "down 4096x14336 BF16, Student-t(5) std 0.02, seed 2",
            "elements": elements, "chunk_elems": chunk_elems, "max_code_len": max_code_len,
            "parallelism": f"replicas x{world}",
            "l2": "no flush: inputs (436 MB) larger than L2 (126 MB)"}


def run_reference(args):
    """The CPU oracle on the host cores, on a bounded sample of the workload."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from exponent_entropy_coding_b200 import synth
    from oracle import ehref
    items = synth.llama8b_block(seed=2, scale=1, count=2)
    sample = items[1][1]           # k_proj, 1024x4096 BF16 = 4,194,304 values
    nbytes = sample.size * 2

    def step():
        c = ehref.compress(ehref.BF16, sample)
        y = ehref.decompress(c)
        return c, y

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        c, y = step()
    dt = (time.perf_counter() - t0) / args.steps
    assert np.array_equal(y, sample)
    v = 2 * nbytes / dt / 1e9
    desc = "oracle compress+decompress of k_proj (1024x4096 BF16, 8.4 MB) per step"
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "GB/s", "n_gpus": args.gpus,
        # `config` names the workload the GPU arm runs; each step of this arm
        # codes only a bounded sample of it (the metric is a rate)
        "sample_per_step": {"tensor": "k_proj", "shape": [1024, 4096], "elements": int(sample.size),
                            "of_workload_elements": 218103808},
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "u16",
        "data": "synthetic", "config": workload_config(args.gpus),
        "cpu_baseline": {"value": v, "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": desc,
                         "cpu": host_cpu_model(), "host_cores": os.cpu_count()},
        "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "size_ratio": (c.stream.size + c.sign_mant.size + 8 * c.chunk_bit_off.size + 256) / nbytes,
    }
    print(json.dumps(line))
    return 0


def cpu_baseline_oracle(items, budget_s=12.0):
    """Single-threaded oracle round trips over the block's matrices until the
    time budget is used (at least one matrix)."""
    from oracle import ehref
    done_bytes, t0, names = 0, time.perf_counter(), []
    for name, x in items:
        c = ehref.compress(ehref.BF16, x)
        y = ehref.decompress(c)
        assert np.array_equal(y, x)
        done_bytes += 2 * x.size * 2
        names.append(name)
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": done_bytes / dt / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"one compress+decompress of {'+'.join(names)} ({done_bytes // 2 / 1e6:.1f} MB BF16)"
                      f" on one host core, {dt:.1f} s"}


_start_barrier = None


def _oracle_worker_init(barrier):
    global _start_barrier
    _start_barrier = barrier


def _oracle_round_trip(index, parts, repeats):
    """Slice `index` of `parts` equal runs of whole chunks of q_proj through
    the oracle as a tensor of its own, timed from a barrier that all workers
    pass together once their inputs exist; returns (BF16 bytes moved both
    ways, start time, end time)."""
    from exponent_entropy_coding_b200 import synth
    from oracle import ehref
    ehref.lib()
    _, x = synth.llama8b_block(seed=2, scale=1, count=1)[0]
    chunks = x.size // 65536
    lo, hi = index * chunks // parts * 65536, (index + 1) * chunks // parts * 65536
    x = np.ascontiguousarray(x[lo:hi])
    _start_barrier.wait()
    t0 = time.perf_counter()
    for _ in range(repeats):
        c = ehref.compress(ehref.BF16, x)
        y = ehref.decompress(c)
    t1 = time.perf_counter()
    assert np.array_equal(y, x)
    return repeats * 2 * 2 * x.size, t0, t1


def cpu_baseline_oracle_parallel(repeats=8):
    """The oracle as it stands on T host cores ("oracle x T"): T spawned
    workers each round-trip an equal run of whole chunks of q_proj (16.8 M
    values) as their own tensor `repeats` times, side by side; the value is
    all their bytes over the time from the common start to the last finish."""
    import multiprocessing as mp
    T = max(1, min(16, os.cpu_count() or 1))
    ctx = mp.get_context("spawn")
    barrier = ctx.Barrier(T)
    with ctx.Pool(T, initializer=_oracle_worker_init, initargs=(barrier,)) as pool:
        res = pool.starmap(_oracle_round_trip, [(i, T, repeats) for i in range(T)], chunksize=1)
    nbytes = sum(r[0] for r in res)
    dt = max(r[2] for r in res) - min(r[1] for r in res)
    return {"value": nbytes / dt / 1e9, "unit": "GB/s", "cores": T, "kind": "oracle",
            "sample": f"q_proj (16.8 M values) in {T} runs of whole chunks, one per process, {repeats} "
                      f"compress+decompress each, started together, {dt:.2f} s"}


def run_ncu_case():
    """Small case for profiler captures: gate_proj alone (117 MB of BF16, more
    than the 126 MB L2 once its compressed form is counted), compressed once
    and decompressed once: three codec kernel launches that matter (hist,
    encode, decode)."""
    import torch

    from exponent_entropy_coding_b200 import exphuff as eh
    from exponent_entropy_coding_b200 import synth
    rng = np.random.default_rng(2)
    x = synth.student_t_bf16((14336, 4096), rng).reshape(-1)
    t = torch.from_numpy(x.view(np.int16)).cuda()
    p = eh.plan(eh.EH_BF16)
    c = eh.compress(t, p)
    y = eh.decompress(c, p)
    torch.cuda.synchronize()
    assert torch.equal(y, t)
    print(json.dumps({"case": "gate_proj 14336x4096", "bits": c.exp_stream_bits,
                      "size_ratio": c.compressed_bytes() / (2 * x.size)}))
    return 0


def run_ncu_pages():
    """Small case for profiler captures of the page store: the K/V workload's
    192 pages (25 MB of BF16) appended once into 28 KB slots with a codebook
    frozen from the first 64 pages, then read back once: one launch each of
    page_bits_kernel, page_encode_kernel and (page mode) decode_kernel."""
    import torch

    from exponent_entropy_coding_b200 import exphuff as eh
    from exponent_entropy_coding_b200 import synth
    dev = torch.device("cuda", 0)
    k = synth.kv_tensor(np.random.default_rng(3), 2, 8192)
    page = 65536
    p = eh.plan(eh.EH_BF16)
    prefill = torch.from_numpy(k[: 64 * page].view(np.int16)).to(dev)
    scratch = eh.alloc_compressed(p, prefill.numel(), dev)
    ws = torch.empty(eh.compress_bound(p, prefill.numel())[2], dtype=torch.uint8, device=dev)
    counts = torch.zeros(256, dtype=torch.int64, device=dev)
    eh.compress_shard_begin(prefill, scratch, counts, p, ws)  # the prefill's exponent counts
    code_len, code = eh.codebook_from_counts(p, counts + 1)
    new = torch.from_numpy(k[64 * page:].view(np.int16)).to(dev)
    n_new = new.numel() // page
    store = eh.PageStore(p, code_len, code, n_slots=n_new, slot_bytes=28 * 1024, raw_cap=n_new, device=dev)
    ids = torch.arange(n_new, dtype=torch.int32, device=dev)
    store.append(new, ids)
    y = store.read(ids)
    torch.cuda.synchronize()
    assert store.status() == eh.EH_OK and torch.equal(y, new)
    print(json.dumps({"case": "K/V page store, 192 pages", "raw_pages": int((store.page_meta < 0).sum())}))
    return 0


def run_all_configs(reps=20):
    """One JSON line per workload (the five of the codec's table): batched
    compress and decompress timed with CUDA events, median of `reps` after 3
    warm-ups, a 256 MB L2 flush before every timed call; algorithmic-byte
    fractions of the measured copy bandwidth; the oracle's round trip of the
    workload's first tensor on one host core beside it."""
    import torch

    from exponent_entropy_coding_b200 import exphuff as eh
    from exponent_entropy_coding_b200 import synth
    from oracle import ehref
    peak, peak_kind = hbm_peak()
    dev = torch.device("cuda", 0)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for name in ("bf16_1m", "fp8_16m", "llama8b_block", "kv_layer", "lm_head"):
        dt, items = synth.workload(name)
        dtype = {"bf16": eh.EH_BF16, "fp8_e4m3": eh.EH_FP8_E4M3}[dt]
        view = np.int16 if dtype == eh.EH_BF16 else np.uint8
        p = eh.plan(dtype)
        xs = [torch.from_numpy(np.ascontiguousarray(x).view(view)).to(dev) for _, x in items]
        outs = [eh.alloc_compressed(p, x.numel(), dev) for x in xs]
        ys = [torch.empty_like(x) for x in xs]
        wsc = torch.empty(eh.compress_batch_workspace(p, [x.numel() for x in xs]), dtype=torch.uint8, device=dev)
        wsd = torch.empty(eh.decompress_workspace(p, len(xs)), dtype=torch.uint8, device=dev)
        bits = torch.zeros(len(xs), dtype=torch.int64, device=dev)
        eh.compress_batch(p, xs, outs, wsc)  # with a host wait: fills the stream sizes
        t_c, t_d = [], []
        for r in range(3 + reps):
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
            flush.zero_()
            ev[0].record()
            eh.compress_batch(p, xs, outs, wsc, bits_dev=bits)
            ev[1].record()
            flush.zero_()
            ev[2].record()
            eh.decompress_batch(p, outs, ys, wsd)
            ev[3].record()
            torch.cuda.synchronize()
            if r >= 3:
                t_c.append(ev[0].elapsed_time(ev[1]) * 1e-3)
                t_d.append(ev[2].elapsed_time(ev[3]) * 1e-3)
        assert eh.get_status(wsd) == eh.EH_OK
        assert all(torch.equal(x, y) for x, y in zip(xs, ys)), name
        n = sum(x.numel() for x in xs)
        nbytes = sum(x.numel() * x.element_size() for x in xs)
        stream_b = sum(o.stream_bytes() for o in outs)
        sm_b = sum(o.sign_mant.numel() for o in outs)
        off_b = sum(8 * o.chunk_bit_off.numel() for o in outs)
        alg = nbytes + sm_b + stream_b + off_b  # each byte once, either direction
        tc, td = statistics.median(t_c), statistics.median(t_d)
        x0 = np.ascontiguousarray(items[0][1])
        a = time.perf_counter()
        c0 = ehref.compress(dtype, x0)
        b_ = time.perf_counter()
        y0 = ehref.decompress(c0)
        e_ = time.perf_counter()
        assert np.array_equal(y0, x0)
        print(json.dumps({
            "config": name, "values": n, "bytes": nbytes,
            "compress_gbs": nbytes / tc / 1e9, "decompress_gbs": nbytes / td / 1e9,
            "compress_frac": alg / tc / 1e9 / peak, "decompress_frac": alg / td / 1e9 / peak,
            "peak_gbs": peak, "peak_kind": peak_kind,
            "compress_us": tc * 1e6, "decompress_us": td * 1e6,
            "size_ratio": sum(o.compressed_bytes() for o in outs) / nbytes,
            "bits_per_exponent": 8 * stream_b / n,
            "oracle": {"compress_gbs": x0.nbytes / (b_ - a) / 1e9, "decompress_gbs": x0.nbytes / (e_ - b_) / 1e9,
                       "cores": 1, "sample": f"{items[0][0]} ({x0.size} values)"},
        }), flush=True)
    return 0


def graph_rate(fn, stream, reps, nbytes):
    """Bytes per second of one call of `fn`, from `reps` calls captured in a
    CUDA graph and replayed between CUDA events (device time only: calls that
    only enqueue small amounts of work would otherwise be timed at the pace of
    the host's Python loop)."""
    import torch

    def loop():
        for _ in range(reps):
            fn()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):  # captured on a side stream
        loop()
    g.replay()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    ev[0].record(stream)
    g.replay()
    ev[1].record(stream)
    torch.cuda.synchronize()
    return nbytes / (ev[0].elapsed_time(ev[1]) / reps * 1e-3) / 1e9


def measure_fp4_scales(eh, synth, items, dev, stream, reps=50):
    """Compress + decompress of the seven matrices' E4M3 block scales (byte
    alphabet), each timed as `reps` calls in a CUDA graph replay; returns GB/s
    of scale bytes and the ratio."""
    import torch
    scales = [synth.nvfp4_block_scales(synth.bf16_bits_to_f32(x)) for _, x in items]
    xs = [torch.from_numpy(s).to(dev) for s in scales]
    p = eh.plan(eh.EH_BYTES)
    outs = [eh.alloc_compressed(p, x.numel(), dev) for x in xs]
    ys = [torch.empty_like(x) for x in xs]
    wsc = torch.empty(eh.compress_batch_workspace(p, [x.numel() for x in xs]), dtype=torch.uint8, device=dev)
    wsd = torch.empty(eh.decompress_workspace(p, len(xs)), dtype=torch.uint8, device=dev)
    bits = torch.zeros(len(xs), dtype=torch.int64, device=dev)
    eh.compress_batch(p, xs, outs, wsc)
    eh.decompress_batch(p, outs, ys, wsd)
    assert eh.get_status(wsd) == eh.EH_OK and all(torch.equal(x, y) for x, y in zip(xs, ys))
    nbytes = sum(x.numel() for x in xs)
    comp = sum(o.compressed_bytes() for o in outs)
    enc = graph_rate(lambda: eh.compress_batch(p, xs, outs, wsc, bits_dev=bits), stream, reps, nbytes)
    dec = graph_rate(lambda: eh.decompress_batch(p, outs, ys, wsd), stream, reps, nbytes)
    assert eh.get_status(wsd) == eh.EH_OK and all(torch.equal(x, y) for x, y in zip(xs, ys))
    return {"kind": f"E4M3 block scales, one per 16 BF16 values of the block; {reps} calls per CUDA graph replay",
            "bytes": nbytes, "encode_gbs": enc, "decode_gbs": dec,
            "size_ratio": comp / nbytes, "bits_per_scale": 8.0 * sum(o.stream_bytes() for o in outs) / nbytes}


def measure_kv_pages(eh, synth, dev, stream, reps=20):
    """Online K/V page store: a K cache of [2, 8192, 8, 128] (256 pages of 64
    tokens); the codebook is frozen from the first 64 pages' exponent counts
    plus one per symbol; the other 192 pages are appended into 28 KB slots in
    one call and read back in one call, with the decode tables prepared once
    (`read_gbs`; building them in every read: `read_gbs_tables_per_call`).
    Device time: `reps` calls of each
    captured in a CUDA graph and replayed between CUDA events (the calls only
    enqueue work, so a Python loop of them measures the host's call overhead
    instead, reported beside as `*_gbs_host_loop`).  BF16 bytes per second."""
    import torch
    rng = np.random.default_rng(3)
    k = synth.kv_tensor(rng, 2, 8192)
    page = 65536
    p = eh.plan(eh.EH_BF16)
    prefill = torch.from_numpy(k[: 64 * page].view(np.int16)).to(dev)
    new = torch.from_numpy(k[64 * page:].view(np.int16)).to(dev)
    n_new = new.numel() // page
    scratch = eh.alloc_compressed(p, prefill.numel(), dev)
    ws = torch.empty(eh.compress_bound(p, prefill.numel())[2], dtype=torch.uint8, device=dev)
    counts = torch.zeros(256, dtype=torch.int64, device=dev)
    eh.compress_shard_begin(prefill, scratch, counts, p, ws)
    code_len, code = eh.codebook_from_counts(p, counts + 1)
    store = eh.PageStore(p, code_len, code, n_slots=n_new, slot_bytes=28 * 1024, raw_cap=n_new, device=dev)
    ids = torch.arange(n_new, dtype=torch.int32, device=dev)
    store.append(new, ids)
    assert store.status() == eh.EH_OK
    y = store.read(ids)
    assert torch.equal(y, new)
    nbytes = 2 * new.numel()

    def timed(fn):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        ev[0].record(stream)
        fn()
        ev[1].record(stream)
        torch.cuda.synchronize()
        return nbytes / (ev[0].elapsed_time(ev[1]) / reps * 1e-3) / 1e9

    def appends():  # on the current stream
        for _ in range(reps):
            store.raw_used.zero_()
            store.append(new, ids)

    def reads():
        for _ in range(reps):
            store.read(ids, out=y, check=False)

    host_append, host_read = timed(appends), timed(reads)

    def append1():
        store.raw_used.zero_()
        store.append(new, ids)
    dev_append = graph_rate(append1, stream, reps, nbytes)
    dev_read_tables = graph_rate(lambda: store.read(ids, out=y, check=False), stream, reps, nbytes)
    store.prepare()  # the frozen codebook's decode tables, built once
    dev_read = graph_rate(lambda: store.read(ids, out=y, check=False), stream, reps, nbytes)
    assert store.status() == eh.EH_OK and torch.equal(y, new)
    meta = store.page_meta.cpu().numpy().view(np.uint32)
    coded = meta[(meta & 0x80000000) == 0]
    return {"kind": "K cache [2, 8192, 8, 128] BF16, 192 pages appended after a 64-page prefill; "
                    f"{reps} calls per CUDA graph replay",
            "append_gbs": dev_append, "read_gbs": dev_read, "read_gbs_tables_per_call": dev_read_tables,
            "append_gbs_host_loop": host_append, "read_gbs_host_loop": host_read,
            "raw_pages": int((meta & 0x80000000).astype(bool).sum()),
            "bits_per_exponent": float(coded.mean()) / page if coded.size else None,
            "slot_bytes": 28 * 1024}


def measure_indexed(eh, p, xs, dev, stream, reps=50):
    """The block with the optional value index (4 bytes per 128 values beside
    the stream): compress writes it, decompress starts every run of 128 values
    at its recorded bit instead of finding code boundaries.  CUDA events;
    GB/s of BF16 bytes, the decoder's fraction of the measured HBM bandwidth
    in algorithmic bytes (the index read counted), and the size ratio with
    the index."""
    import torch
    outs = [eh.alloc_compressed(p, x.numel(), dev, index=True) for x in xs]
    ys = [torch.empty_like(x) for x in xs]
    wsc = torch.empty(eh.compress_batch_workspace(p, [x.numel() for x in xs]), dtype=torch.uint8, device=dev)
    wsd = torch.empty(eh.decompress_workspace(p, len(xs)), dtype=torch.uint8, device=dev)
    bits = torch.zeros(len(xs), dtype=torch.int64, device=dev)
    eh.compress_batch(p, xs, outs, wsc)
    eh.decompress_batch(p, outs, ys, wsd)
    assert eh.get_status(wsd) == eh.EH_OK and all(torch.equal(x, y) for x, y in zip(xs, ys))
    in_bytes = sum(2 * x.numel() for x in xs)
    comp = sum(o.compressed_bytes() for o in outs)
    alg = sum(o.stream_bytes() + o.sign_mant.numel() + 8 * o.chunk_bit_off.numel() + 4 * o.value_index.numel()
              for o in outs) + in_bytes
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    for _ in range(3):
        eh.compress_batch(p, xs, outs, wsc, bits_dev=bits)
        eh.decompress_batch(p, outs, ys, wsd)
    ev[0].record(stream)
    for _ in range(reps):
        eh.compress_batch(p, xs, outs, wsc, bits_dev=bits)
    ev[1].record(stream)
    for _ in range(reps):
        eh.decompress_batch(p, outs, ys, wsd)
    ev[2].record(stream)
    torch.cuda.synchronize()
    assert eh.get_status(wsd) == eh.EH_OK and all(torch.equal(x, y) for x, y in zip(xs, ys))
    enc = ev[0].elapsed_time(ev[1]) / reps * 1e-3
    dec = ev[1].elapsed_time(ev[2]) / reps * 1e-3
    peak, _ = hbm_peak()
    return {"kind": "value index beside the stream (bit offset of every 128th value of each chunk)",
            "encode_gbs": in_bytes / enc / 1e9, "decode_gbs": in_bytes / dec / 1e9,
            "decode_frac": alg / dec / 1e9 / peak, "size_ratio": comp / in_bytes}


def measure_zipfloat(eh, xs, dev, stream, reps=20):
    """The ZipFloat comparison codec on the same block (seven calls each way
    per repetition, CUDA events): GB/s of BF16 bytes and the size ratio."""
    import torch
    cs = [eh.zf_compress(x) for x in xs]
    ys = [torch.empty_like(x) for x in xs]
    for c, x, y in zip(cs, xs, ys):
        eh.zf_decompress(c, out=y)
        assert torch.equal(x, y)
    nbytes = sum(2 * x.numel() for x in xs)
    comp = sum(c.compressed_bytes() for c in cs)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    ev[0].record(stream)
    for _ in range(reps):
        for c, x in zip(cs, xs):
            eh.zf_compress(x, out=c, wait=False)
    ev[1].record(stream)
    for _ in range(reps):
        for c, y in zip(cs, ys):
            eh.zf_decompress(c, out=y, check=False)
    ev[2].record(stream)
    torch.cuda.synchronize()
    enc = ev[0].elapsed_time(ev[1]) / reps
    dec = ev[1].elapsed_time(ev[2]) / reps
    return {"kind": "ZipFloat comparison codec (blocks of 2048, l_b = MD - 6, 3 bit planes, 16-bit records)",
            "encode_gbs": nbytes / (enc * 1e-3) / 1e9, "decode_gbs": nbytes / (dec * 1e-3) / 1e9,
            "size_ratio": comp / nbytes,
            "records_per_value": sum(c.n_records for c in cs) / (nbytes / 2)}


def measure_prefetch(eh, xs, outs, p, dev, tokens, layers=8, depth=2, max_ctas=0, reps=3):
    """Linear layers of `layers` Llama-3.1-8B blocks run on `tokens` rows of
    activations (y = x @ W^T for q, k, v, o, gate, up, down; every layer reuses
    the one compressed block).  Three ways, each timed with CUDA events on the
    consumer stream (median of `reps`):
      resident   the uncompressed weights stay in HBM;
      serial     each block is decompressed, then its GEMMs run, one stream;
      prefetch   the block for layer l+depth is decompressed on a decode
                 stream into a ring slot while layers l..l+depth-1 compute.
    The outputs of the last layer are checked equal across the three."""
    import torch
    cons = torch.cuda.current_stream()
    torch.manual_seed(0)
    shapes = [(x.numel() // (4096 if i < 6 else 14336), 4096 if i < 6 else 14336) for i, x in enumerate(xs)]
    acts = [torch.randn(tokens, k, device=dev).to(torch.bfloat16) for _, k in shapes]
    ws_res = [x.view(torch.bfloat16).view(r, k) for x, (r, k) in zip(xs, shapes)]
    slot_bytes = sum((2 * x.numel() + 255) // 256 * 256 for x in xs)
    pf = eh.Prefetcher(p, depth, slot_bytes, dev, max_ctas=max_ctas)
    serial_buf = [torch.empty_like(x) for x in xs]
    wsd = torch.empty(eh.decompress_workspace(p, len(xs)), dtype=torch.uint8, device=dev)

    def gemms(ws):
        return [a @ w.t() for a, w in zip(acts, ws)]

    def run_resident():
        for _ in range(layers):
            ys = gemms(ws_res)
        return ys

    def run_serial():
        for _ in range(layers):
            eh.decompress_batch(p, outs, serial_buf, wsd)
            ys = gemms([b.view(torch.bfloat16).view(r, k) for b, (r, k) in zip(serial_buf, shapes)])
        return ys

    def run_prefetch(start):
        pf.stream.wait_event(start)
        pending = [pf.submit(outs) for _ in range(min(depth, layers))]
        for l in range(layers):
            slot, views = pending.pop(0)
            pf.acquire(slot, cons)
            ys = gemms([v.view(torch.bfloat16).view(r, k) for v, (r, k) in zip(views, shapes)])
            pf.release(slot, cons)
            if l + depth < layers:
                pending.append(pf.submit(outs))
        return ys

    times = {"resident": [], "serial": [], "prefetch": []}
    results = {}
    for rep in range(reps + 1):  # the first round warms up
        for name in times:
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(cons)
            ys = run_prefetch(e0) if name == "prefetch" else (run_serial() if name == "serial" else run_resident())
            e1.record(cons)
            torch.cuda.synchronize()
            if rep:
                times[name].append(e0.elapsed_time(e1))
            results[name] = ys
    for s in range(depth):
        assert pf.status(s) == eh.EH_OK
    same = all(torch.equal(a, b) and torch.equal(a, c)
               for a, b, c in zip(results["resident"], results["serial"], results["prefetch"]))
    pf.close()
    med = {k: statistics.median(v) for k, v in times.items()}
    return {"tokens": tokens, "layers": layers, "depth": depth, "decode_ctas": max_ctas or "all",
            "resident_ms": med["resident"], "serial_ms": med["serial"], "prefetch_ms": med["prefetch"],
            "prefetch_over_resident": med["prefetch"] / med["resident"],
            "serial_over_resident": med["serial"] / med["resident"], "outputs_equal": same}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--no-side", action="store_true",
                    help="skip the side measurements (FP4 scales, K/V pages, ZipFloat, prefetch ring)")
    ap.add_argument("--all-configs", action="store_true",
                    help="one line per workload of the codec's table (compress/decompress, fractions, oracle)")
    ap.add_argument("--ncu-case", nargs="?", const="gate", choices=["gate", "pages"],
                    help="for ncu captures: one compress + one decompress of gate_proj (14336x4096), "
                         "or (pages) one append + one read of the 192-page K/V store")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.ncu_case == "pages":
        return run_ncu_pages()
    if args.ncu_case:
        return run_ncu_case()
    if args.all_configs:
        return run_all_configs()

    import torch
    import torch.distributed as dist

    from exponent_entropy_coding_b200 import exphuff as eh
    from exponent_entropy_coding_b200 import synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300))
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()

    items = synth.llama8b_block(seed=2, scale=1)
    ns = [x.size for _, x in items]
    in_bytes = 2 * sum(ns)
    xs_host = [torch.from_numpy(x.view(np.int16)).pin_memory() for _, x in items]
    xs = [h.to(dev) for h in xs_host]
    p = eh.plan(eh.EH_BF16)
    outs = [eh.alloc_compressed(p, n, dev) for n in ns]
    ys = [torch.empty_like(x) for x in xs]
    wsc = torch.empty(eh.compress_batch_workspace(p, ns), dtype=torch.uint8, device=dev)
    wsd = torch.empty(eh.decompress_workspace(p, len(xs)), dtype=torch.uint8, device=dev)
    bits = torch.zeros(len(xs), dtype=torch.int64, device=dev)

    # first pass: exactness and sizes
    eh.compress_batch(p, xs, outs, wsc)
    eh.decompress_batch(p, outs, ys, wsd)
    assert eh.get_status(wsd) == eh.EH_OK
    assert all(torch.equal(x, y) for x, y in zip(xs, ys)), "round trip mismatch"
    stream_bytes = sum(o.stream_bytes() for o in outs)
    comp_bytes = sum(o.compressed_bytes() for o in outs)
    sm_bytes = sum(o.sign_mant.numel() for o in outs)
    off_bytes = sum(8 * o.chunk_bit_off.numel() for o in outs)

    n_ev = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n_ev)]

    def step(i=None):
        if i is not None:
            ev[i][0].record(stream)
        eh.compress_batch(p, xs, outs, wsc, bits_dev=bits)
        if i is not None:
            ev[i][1].record(stream)
        eh.decompress_batch(p, outs, ys, wsd)
        if i is not None:
            ev[i][2].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        t_start.record(stream)
        for i in range(args.steps):
            step(i)
        t_end.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms = t_start.elapsed_time(t_end) / args.steps
    enc_ms = statistics.mean(a.elapsed_time(b) for a, b, _ in ev)
    dec_ms = statistics.mean(b.elapsed_time(c) for _, b, c in ev)
    assert eh.get_status(wsd) == eh.EH_OK
    assert all(torch.equal(x, y) for x, y in zip(xs, ys)), "round trip mismatch after timing"
    if world > 1:
        t = torch.tensor([ms, enc_ms, dec_ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms, enc_ms, dec_ms = t.tolist()

    # end to end through the public API: pinned host -> device copy of the
    # block, compress (host wait for the bit counts), decompress, status read
    e2e_steps = max(1, args.e2e_steps)
    for _ in range(2):
        for h, x in zip(xs_host, xs):
            x.copy_(h, non_blocking=True)
        eh.compress_batch(p, xs, outs, wsc)
        eh.decompress_batch(p, outs, ys, wsd)
        eh.get_status(wsd)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        for h, x in zip(xs_host, xs):
            x.copy_(h, non_blocking=True)
        eh.compress_batch(p, xs, outs, wsc)
        eh.decompress_batch(p, outs, ys, wsd)
        st = eh.get_status(wsd)
        assert st == eh.EH_OK
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    if world > 1:
        t = torch.tensor([e2e_ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_ms = t.item()
        dist.barrier()

    # side measurement (outside the timed region): the codec on the block's
    # FP4 block scale factors (NVFP4-style E4M3 scales, one per 16 values)
    fp4 = kv_pages = prefetch = zipfloat = indexed = None
    if not args.no_side:
        indexed = measure_indexed(eh, p, xs, dev, stream)
        fp4 = measure_fp4_scales(eh, synth, items, dev, stream)
        kv_pages = measure_kv_pages(eh, synth, dev, stream)
        # decompression into the operand buffers of the next GEMMs (prefetch ring)
        prefetch = [measure_prefetch(eh, xs, outs, p, dev, t) for t in (1, 8192)]
        zipfloat = measure_zipfloat(eh, xs, dev, stream)

    if rank == 0:
        peak, peak_kind = hbm_peak()
        value = world * 2 * in_bytes / (ms * 1e-3) / 1e9
        enc_gbs = in_bytes / (enc_ms * 1e-3) / 1e9
        dec_gbs = in_bytes / (dec_ms * 1e-3) / 1e9
        # algorithmic bytes, each byte counted once
        dec_alg = stream_bytes + sm_bytes + off_bytes + in_bytes
        enc_alg = in_bytes + sm_bytes + stream_bytes + off_bytes
        dec_achieved = dec_alg / (dec_ms * 1e-3) / 1e9
        enc_achieved = enc_alg / (enc_ms * 1e-3) / 1e9
        traffic = None
        if DECODE_TRAFFIC["bytes"] and DECODE_TRAFFIC["source_sha"] == decoder_source_sha():
            traffic = DECODE_TRAFFIC["bytes"]
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "u16",
            "data": "synthetic",
            "config": workload_config(world, sum(ns), p.chunk_elems, p.max_code_len),
            "decode_gbs": dec_gbs, "encode_gbs": enc_gbs,
            "pct_hbm": {"decode": dec_achieved / peak, "encode": enc_achieved / peak,
                        # the compressor's real traffic reads the input twice (the
                        # histogram must be complete before any code is known)
                        "encode_with_second_read": (enc_alg + in_bytes) / (enc_ms * 1e-3) / 1e9 / peak,
                        "peak_gbs": peak, "peak_kind": peak_kind},
            "size_ratio": comp_bytes / in_bytes,
            "bits_per_exponent": 8 * stream_bytes / sum(ns),
            "roofline": {"bound": "hbm", "kernel": "decode (tables + decode launch)",
                         "achieved": dec_achieved, "peak": peak, "unit": "GB/s",
                         "frac": dec_achieved / peak, "traffic": traffic,
                         "algorithmic_bytes": dec_alg, "peak_kind": peak_kind},
            "e2e": {"value": world * 2 * in_bytes / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
                    "h2d_bytes_per_step": in_bytes, "d2h_bytes_per_step": 8 + 8 * len(ns) + 4,
                    "ms_per_step": e2e_ms},
            "gpu_launches": 6 * args.steps,
            "fp4_scales": fp4,
            "kv_pages": kv_pages,
            "indexed": indexed,
            "zipfloat": zipfloat,
            "prefetch": {"workload": "8 layers of Llama-3.1-8B block linears (q,k,v,o,gate,up,down) "
                                     "on `tokens` BF16 rows; weights decoded into a 2-slot ring",
                         "runs": prefetch},
            "clocks": clk.summary(),
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline_oracle(items)
            line["cpu_baseline_parallel"] = cpu_baseline_oracle_parallel()
            for k in ("cpu_baseline", "cpu_baseline_parallel"):
                if isinstance(line.get(k), dict):
                    line[k]["cpu"] = host_cpu_model()
                    line[k]["host_cores"] = os.cpu_count()
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
