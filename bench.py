"""Benchmark: int4-KV decode attention on B200 (effective HBM GB/s and tokens/s).

One step is the whole hot path on one batch: quantise-append one new K/V token
per sequence (SRHT + per-group abs-max int4 + nibble pack) and one decode query
per sequence over its packed cache (rotated query, split-K online softmax on
tensor cores, merge + inverse SRHT). The default workload is the 32-sequence
ragged serving batch (contexts U{1024..32768}, 32 q / 8 kv heads, D = 128,
bf16 inputs); ``--workload`` picks another recipe from
``compressed_domain_attention_b200.synthetic``.

Timing: W warm-up steps, then K steps between a barrier + synchronize on both
sides, CUDA events on the launching stream, max over ranks. The packed cache
(about 1.2 GB for the default workload) is larger than the 126 MB L2, so no L2
flush is needed. ``--gpus N`` (under torchrun) runs N independent replicas: the
path has no exchange step, so there is no collective on the data path.

The default line also carries ``long_context``: the same step timed on the
131072-token Llama-3.1-70B-shaped context (64 q / 8 kv heads, query groups of
8), with its own split-K roofline record (``--no-long-context`` skips it).

``--impl reference`` times the CPU oracle (plain single-threaded C++) on a
bounded sample of the same workload on the host cores.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "int4-KV decode attention effective HBM GB/s (packed K/V codes + fp16 scales per step)"
UNIT = "GB/s"


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["tq", "reference"], default="tq")
    ap.add_argument("--workload", default="ragged_serving",
                    choices=["ragged_serving", "llama31_70b_long", "llama3_8b_layer", "tiny_single_head"])
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the oracle timing leg")
    ap.add_argument("--no-clocks", action="store_true", help="skip nvidia-smi clock sampling")
    ap.add_argument("--no-long-context", action="store_true",
                    help="skip the 131072-token long-context sub-record of the default line")
    ap.add_argument("--no-references", action="store_true",
                    help="skip the quantise-throughput, bf16 dense-KV and dequantise-then-attend reference points")
    ap.add_argument("--k-format", choices=list(FORMATS), default="int4",
                    help="cache format: int4 K and V (symmetric cache); binary16 K in the original domain with "
                         "int4 V (the asymmetric cache of the mlxcel guide's recommended mode); or 'delegated', "
                         "binary16 K with a binary16 V hot tail folded into int4 V (the guide's delegated mode)")
    ap.add_argument("--lambda", dest="lam", action="store_true",
                    help="write and read the cache with seeded per-channel lambda vectors (K with int4 K, and V)")
    ap.add_argument("--sparse-v", type=float, default=0.0, metavar="TAU",
                    help="sparse-V threshold of the decode (0 = exact attention; the mlxcel guide's default is 1e-6)")
    ap.add_argument("--paged", type=int, default=0, metavar="P",
                    help="paged storage with P-token pages (a seeded random permutation of the pool's pages); "
                         "int4 and fp16 formats")
    ap.add_argument("--sweep", action="store_true",
                    help="per-configuration report instead of the step benchmark: decode and prefill-quantise "
                         "times (median, p10, p90; cold L2, and warm L2 where the cache fits) for every workload "
                         "shape, one JSON line each")
    return ap.parse_args(argv)


def get_workload(name):
    from compressed_domain_attention_b200 import synthetic as syn
    return {"ragged_serving": syn.ragged_serving, "llama31_70b_long": syn.llama31_70b_long,
            "llama3_8b_layer": syn.llama3_8b_layer, "tiny_single_head": syn.tiny_single_head}[name]()


# ----------------------------------------------------------------------------- algorithmic bytes

FORMATS = ("int4", "fp16", "delegated")


def delegated_window():
    from compressed_domain_attention_b200 import synthetic as syn
    return syn.DELEGATED_WINDOW, syn.DELEGATED_FOLD


def bench_lambdas(D, fmt, device):
    """Seeded per-channel lambda vectors exp(U(-1, 1)) for K (int4 K only) and V."""
    import torch
    g = torch.Generator("cpu").manual_seed(1234)
    lk = torch.exp(torch.rand(D, generator=g) * 2 - 1).float()
    lv = torch.exp(torch.rand(D, generator=g) * 2 - 1).float()
    return (lk.to(device) if fmt == "int4" else None), lv.to(device)


def cold_count(n, fmt):
    """Tokens of an n-token sequence held as int4 V codes: all of them, except in the delegated cache,
    whose most recent tokens (between W - F + 1 and W once n > W) stay binary16 in the hot tail."""
    if fmt != "delegated":
        return n
    W, F = delegated_window()
    return 0 if n <= W else (n - W + F - 1) // F * F


def split_bytes(w, lens, fmt="int4"):
    """Cache bytes the split-K kernel reads: per cold token.kv-head, packed V codes + binary16 scales
    (D/2 + D/16), and the same again for int4 K or 2D for binary16 K."""
    D = w.head_dim
    v = D // 2 + 2 * (D // 32)
    k = v if fmt == "int4" else 2 * D
    return sum(cold_count(n, fmt) for n in lens) * w.n_kv_heads * (v + k)


def decode_bytes(w, lens, fmt="int4"):
    """Cache bytes the decode reads per step: the split-K kernel's, plus (delegated cache) the hot
    tokens' binary16 K and V rows, which the merge kernel reads."""
    D = w.head_dim
    hot = sum(n - cold_count(n, fmt) for n in lens)
    return split_bytes(w, lens, fmt) + hot * w.n_kv_heads * 4 * D


def append_bytes(w, in_bytes=2, fmt="int4", lens0=None):
    """Append traffic per step: raw K/V in, packed codes and scales (or binary16 K / binary16 V tail) out;
    for the delegated cache also the tokens that fold out of the tail (binary16 in, codes and scales out)."""
    D = w.head_dim
    code = D // 2 + 2 * (D // 32)
    v_vec = D * in_bytes + (2 * D if fmt == "delegated" else code)
    k_vec = D * in_bytes + (code if fmt == "int4" else 2 * D)
    total = w.batch * w.n_append * w.n_kv_heads * (v_vec + k_vec)
    if fmt == "delegated":
        lens0 = w.seq_lens if lens0 is None else lens0
        folds = sum(cold_count(n + w.n_append, fmt) - cold_count(n, fmt) for n in lens0)
        total += folds * w.n_kv_heads * (2 * D + code)
    return total


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def load_traffic(kernel_key):
    """ncu DRAM bytes per launch recorded in profiles/ for the current kernel source (else None)."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    src = os.path.join(ROOT, "compressed_domain_attention_b200", "csrc", "tq_decode.cu")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    digest = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    ent = rec.get(kernel_key)
    if not ent or ent.get("source_sha256_16") != digest:
        return None
    return ent.get("dram_bytes_per_full_launch")


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    def __init__(self, device_index):
        self.idx = device_index
        self.samples = []
        self.proc = None
        self.thread = None

    def start(self):
        q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
             "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
             "clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.idx), f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 7:
                self.samples.append(parts)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        if not self.samples:
            return None
        sm = []
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        mx = None
        for p in self.samples:
            try:
                sm.append(float(p[0]))
                mx = float(p[1])
            except ValueError:
                continue
            for n, v in zip(names, p[3:7]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- distributed plumbing

def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def init_dist(backend):
    import torch.distributed as dist
    ws, rank, _ = dist_env()
    if ws > 1 and not dist.is_initialized():
        import datetime
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return ws, rank


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_initialized():
        if device is not None and dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def max_over_ranks(value, device=None):
    """Max of a float over all ranks (identity on one process)."""
    import torch
    import torch.distributed as dist
    if not dist.is_initialized():
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value, device=None):
    import torch
    import torch.distributed as dist
    if not dist.is_initialized():
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def assemble_line(*, n_gpus, steps, warmup, total_bytes_all_ranks, max_time_s, workload, extra):
    """The JSON result line (value = whole-job GB/s over all ranks)."""
    value = total_bytes_all_ranks / max_time_s / 1e9
    line = {"metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": n_gpus, "steps": steps,
            "warmup": warmup, "ms_per_step": round(max_time_s / steps * 1e3, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "int4 codes, f16 tensor-core operands, f32 accumulate",
            "data": "synthetic (seeded; outlier-channel K, no weights or datasets)", "config": workload}
    line.update(extra)
    return line


# ----------------------------------------------------------------------------- CPU oracle timing

def oracle_sample(w, target_tokens, longest_first=False):
    """Sequences for a bounded oracle sample: up to about `target_tokens` KV tokens."""
    order = sorted(range(w.batch), key=lambda b: w.seq_lens[b], reverse=longest_first)
    picked, tot = [], 0
    for b in order:
        if tot >= target_tokens and picked:
            break
        picked.append(b)
        tot += w.seq_lens[b]
    return sorted(picked)


class OracleStep:
    """The oracle's version of one step (append one token per sequence, decode) on a sample of sequences.

    The sample's caches are encoded once at construction (untimed); each step
    re-appends the new token at position len_b and decodes over len_b + 1.
    """

    def __init__(self, w, tensors, seqs, fmt="int4", lam=False, tau=0.0):
        import numpy as np
        import oracle
        from compressed_domain_attention_b200 import synthetic as syn
        self.oracle, self.np = oracle, np
        D, H = w.head_dim, w.n_kv_heads
        self.w, self.seqs, self.fmt, self.tau = w, seqs, fmt, tau
        self.lk = self.lv = None
        if lam:
            lk, lv = bench_lambdas(D, fmt, "cpu")
            self.lk = None if lk is None else lk.numpy()
            self.lv = lv.numpy()
        self.s = oracle.sign_vector(0, D)
        n = len(seqs)
        cap = max(w.seq_lens[b] for b in seqs) + 1
        if fmt == "int4":
            self.kc, self.ks = oracle.new_cache(n, cap, H, D)
        else:
            self.kc, self.ks = oracle.new_k16_cache(n, cap, H, D), None
        self.vc, self.vs = oracle.new_cache(n, cap, H, D)
        self.W, self.F = delegated_window() if fmt == "delegated" else (0, 0)
        self.tail = oracle.new_tail(n, self.W, H, D) if fmt == "delegated" else None
        for i, b in enumerate(seqs):
            k = tensors.k[b].float().cpu().numpy()[None]
            v = tensors.v[b].float().cpu().numpy()[None]
            self._append(i, i + 1, k, v, np.zeros(1, np.int32))
        self.q = np.ascontiguousarray(tensors.q[seqs].float().cpu().numpy())
        self.kn = np.ascontiguousarray(tensors.k_new[seqs].float().cpu().numpy())
        self.vn = np.ascontiguousarray(tensors.v_new[seqs].float().cpu().numpy())
        self.lens = np.array([w.seq_lens[b] for b in seqs], np.int32)
        sub = syn.Workload(w.name, n, w.n_q_heads, H, D, [w.seq_lens[b] for b in seqs], w.dtype, w.seed, n_append=1)
        self.nbytes = decode_bytes(sub, [L + 1 for L in sub.seq_lens], fmt) + append_bytes(sub, fmt=fmt)
        self.ntok = int(self.lens.sum()) + n

    def _append(self, i0, i1, k, v, start):
        sl = slice(i0, i1)
        if self.fmt == "delegated":
            self.oracle.append_delegated(self.s, k, v, start, self.W, self.F, self.kc[sl], self.vc[sl], self.vs[sl],
                                         self.tail[sl])
        elif self.fmt == "fp16":
            if self.lv is not None:  # binary16 K as numpy rounds it, V through the lambda encoder
                np_ = self.np
                n = k.shape[1]
                for j, b in enumerate(range(i0, i1)):
                    p0 = int(start[j])
                    self.kc[b, p0:p0 + n] = k[j].astype(np_.float16).view(np_.uint16)
                kd, ksd = self.oracle.new_cache(i1 - i0, self.vc.shape[1], self.vc.shape[2], self.w.head_dim)
                self.oracle.quantize_append_lambda(self.s, k, v, start, None, self.lv, kd, ksd, self.vc[sl],
                                                   self.vs[sl])
            else:
                self.oracle.quantize_append_kf16(self.s, k, v, start, self.kc[sl], self.vc[sl], self.vs[sl])
        elif self.lk is not None or self.lv is not None:
            self.oracle.quantize_append_lambda(self.s, k, v, start, self.lk, self.lv, self.kc[sl], self.ks[sl],
                                               self.vc[sl], self.vs[sl])
        else:
            self.oracle.quantize_append(self.s, k, v, start, self.kc[sl], self.ks[sl], self.vc[sl], self.vs[sl])

    def _decode(self, i0, i1, q, lens):
        sl = slice(i0, i1)
        if self.fmt == "delegated":
            self.oracle.decode_attention_delegated(self.s, q, lens, self.kc[sl], self.vc[sl], self.vs[sl],
                                                   self.tail[sl], self.W, self.F, self.w.scale)
        elif self.lk is not None or self.lv is not None or self.tau > 0:
            kf = self.fmt == "fp16"
            self.oracle.decode_attention_ext(self.s, q, lens, None if kf else self.kc[sl],
                                             None if kf else self.ks[sl], self.vc[sl], self.vs[sl], self.w.scale,
                                             self.lk, self.lv, self.tau, k_f16=self.kc[sl] if kf else None)
        elif self.fmt == "fp16":
            self.oracle.decode_attention_kf16(self.s, q, lens, self.kc[sl], self.vc[sl], self.vs[sl], self.w.scale)
        else:
            self.oracle.decode_attention(self.s, q, lens, self.kc[sl], self.ks[sl], self.vc[sl], self.vs[sl],
                                         self.w.scale)

    def run(self):
        n = len(self.seqs)
        t0 = time.perf_counter()
        self._append(0, n, self.kn, self.vn, self.lens)
        self._decode(0, n, self.q, self.lens + 1)
        return time.perf_counter() - t0

    def run_parallel(self, threads):
        """The same step with independent sequences spread over host threads.

        Each thread calls the unchanged oracle on one sequence's slices; the C++
        calls release the interpreter lock, so the threads run on separate cores.
        """
        from concurrent.futures import ThreadPoolExecutor
        o, n = self.oracle, len(self.seqs)

        def one(i):
            sl = slice(i, i + 1)
            self._append(i, i + 1, self.kn[sl], self.vn[sl], self.lens[sl])
            self._decode(i, i + 1, self.q[sl], self.lens[sl] + 1)

        with ThreadPoolExecutor(max_workers=threads) as ex:
            t0 = time.perf_counter()
            list(ex.map(one, range(n)))
            return time.perf_counter() - t0


def cpu_model():
    """The host CPU's model name (Linux /proc/cpuinfo), or the platform's processor string."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover - non-Linux hosts
        return os.cpu_count() or 1


def cpu_baseline(w, tensors, target_tokens, fmt="int4", lam=False, tau=0.0):
    seqs = oracle_sample(w, target_tokens)
    o = OracleStep(w, tensors, seqs, fmt, lam, tau)
    dt = o.run()
    line = {"value": round(o.nbytes / dt / 1e9, 4), "unit": UNIT, "cores": 1, "kind": "oracle",
            "cpu_model": cpu_model(), "host_cores": host_cores(),
            "sample": f"one step (append + decode) on {len(seqs)} of {w.batch} sequences "
                      f"({o.ntok} KV tokens x {w.n_q_heads} q heads), single-threaded C++ oracle, {dt:.2f} s",
            "seconds": round(dt, 3)}
    cores = host_cores()
    if cores > 1 and len(seqs) > 1:
        dtp = o.run_parallel(min(cores, len(seqs)))
        line["parallel"] = {"value": round(o.nbytes / dtp / 1e9, 4), "unit": UNIT,
                            "cores": min(cores, len(seqs)), "host_cores": cores, "seconds": round(dtp, 3),
                            "how": "the same sample, one sequence per task on a thread pool over the unchanged "
                                   "oracle (its C++ calls run outside the interpreter lock)"}
    return line


# ----------------------------------------------------------------------------- same-run reference points

def _time_cold(fn, reps, flush, stream):
    """Median device time (ms) of fn() with the L2 flushed (a buffer > L2 rewritten) before each rep."""
    import torch
    ts = []
    for _ in range(reps):
        flush.add_(1)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    return statistics.median(ts)


def reference_points(w, t, L, kc, ks, vc, vs, lens1, q, dev, stream, args, fmt="int4"):
    """Quantise throughput, the bf16 dense-KV decode and dequantise-then-attend, on this GPU and workload."""
    import torch
    import torch.nn.functional as F
    from compressed_domain_attention_b200 import synthetic as syn
    from compressed_domain_attention_b200 import tq
    out = {}
    flush = torch.zeros(64 << 20, dtype=torch.float32, device=dev)  # 256 MB > 126 MB L2
    # 1. quantise-append throughput: a 4096-token prefill of one sequence (all kv heads, K and V)
    pw = syn.Workload("prefill_4096", 1, w.n_q_heads, w.n_kv_heads, w.head_dim, [4096], w.dtype, w.seed + 100)
    pt = syn.generate(pw, device="cuda")
    pl = tq.tq_cache_layout(1, 4096, w.n_kv_heads, w.n_q_heads, w.head_dim)
    pkc, pks, pvc, pvs = tq.alloc_cache(pl, dev)
    zero = torch.zeros(1, dtype=torch.int32, device=dev)
    pk, pv = pt.k[0][None].contiguous(), pt.v[0][None].contiguous()

    def prefill():
        tq.tq_quantize_append(pl, pk, pv, 4096, zero, pkc, pks, pvc, pvs, None, stream)

    for _ in range(3):
        prefill()
    ms = _time_cold(prefill, 20, flush, stream)
    vecs = 2 * 4096 * w.n_kv_heads
    per_vec = w.head_dim * pk.element_size() + w.head_dim // 2 + 2 * (w.head_dim // 32)
    out["quantize"] = {"workload": f"4096-token prefill of one sequence, {w.n_kv_heads} kv heads, K and V "
                                   f"({vecs} vectors, {pk.dtype})".replace("torch.", ""),
                       "ms": round(ms, 4), "vectors_per_s": round(vecs / ms * 1e3, 1),
                       "gb_per_s": round(vecs * per_vec / ms / 1e6, 1), "l2": "flushed before each rep"}
    del pkc, pks, pvc, pvs, pk, pv, pt
    # 2. bf16 dense-KV decode on the same (unquantised) data: torch SDPA per sequence, in a CUDA graph
    if w.dtype != torch.float32 and not args.no_references:
        ks_d = [t.k[b].permute(1, 0, 2).contiguous()[None] for b in range(w.batch)]  # [1][Hkv][L][D]
        vs_d = [t.v[b].permute(1, 0, 2).contiguous()[None] for b in range(w.batch)]
        qd = q.view(w.batch, w.n_q_heads, 1, w.head_dim)
        outs = [None] * w.batch

        def dense():
            for b in range(w.batch):
                outs[b] = F.scaled_dot_product_attention(qd[b:b + 1], ks_d[b], vs_d[b], scale=w.scale,
                                                         enable_gqa=True)

        try:
            dense()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                dense()
            ms_d = _time_cold(g.replay, 10, flush, stream)
            dbytes = 2 * 2 * w.head_dim * w.n_kv_heads * sum(w.seq_lens)
            out["bf16_dense_decode"] = {
                "impl": "torch.nn.functional.scaled_dot_product_attention (enable_gqa), one call per sequence "
                        "in a CUDA graph, bf16 K/V on the same data",
                "ms": round(ms_d, 4), "gb_per_s": round(dbytes / ms_d / 1e6, 1),
                "bytes": dbytes, "l2": "flushed before each rep"}
            del g
        except RuntimeError as e:  # noqa: BLE001
            out["bf16_dense_decode"] = {"unavailable": str(e).splitlines()[0][:200]}
        del ks_d, vs_d
        torch.cuda.empty_cache()
    # 3. dequantise-then-attend (the comparison category of the Open-TQ-Metal abstract):
    #    tq_dequantize_debug to dense fp32 K/V in the original domain, then SDPA per sequence
    if (not args.no_references and fmt == "int4"
            and w.batch * L.max_seq * w.n_kv_heads * w.head_dim * 4 * 2 < 24e9):
        Kd = torch.empty((w.batch, L.max_seq, w.n_kv_heads, w.head_dim), dtype=torch.float32, device=dev)
        Vd = torch.empty_like(Kd)
        qf = q.float().view(w.batch, w.n_q_heads, 1, w.head_dim)
        lens_list = [x + w.n_append for x in w.seq_lens]

        def deq_attend():
            tq.tq_dequantize_debug(L, kc, ks, lens1, True, Kd, stream)
            tq.tq_dequantize_debug(L, vc, vs, lens1, True, Vd, stream)
            for b in range(w.batch):
                n = lens_list[b]
                F.scaled_dot_product_attention(qf[b:b + 1], Kd[b, :n].permute(1, 0, 2)[None],
                                               Vd[b, :n].permute(1, 0, 2)[None], scale=w.scale, enable_gqa=True)

        try:
            deq_attend()
            ms_q = _time_cold(deq_attend, 5, flush, stream)
            out["dequantize_then_attend"] = {
                "impl": "tq_dequantize_debug (fp32, original domain) + torch SDPA per sequence",
                "ms": round(ms_q, 3)}
        except RuntimeError as e:  # noqa: BLE001
            out["dequantize_then_attend"] = {"unavailable": str(e).splitlines()[0][:200]}
        del Kd, Vd
        torch.cuda.empty_cache()
    return out



# ----------------------------------------------------------------------------- the cache on the device

class DeviceCache:
    """One cache format in device memory, driven through the library's C ABI (tq.py)."""

    def __init__(self, w, cap, fmt, dev, lam=False, tau=0.0, page=0):
        import torch
        from compressed_domain_attention_b200 import tq
        self.tq, self.fmt, self.tau, self.page = tq, fmt, tau, page
        self.lk, self.lv = bench_lambdas(w.head_dim, fmt, dev) if lam else (None, None)
        shape = (cap, w.n_kv_heads, w.n_q_heads, w.head_dim)
        if page:
            kfmt = tq.TQ_K_INT4 if fmt == "int4" else tq.TQ_K_FP16
            max_pages = -(-cap // page)
            n_pages = w.batch * max_pages
            self.L = tq.tq_cache_layout_paged(w.batch, *shape, kfmt, page, n_pages)
            self.l1 = tq.tq_cache_layout_paged(1, *shape, kfmt, page, n_pages)
            g = torch.Generator("cpu").manual_seed(77)  # pages scattered over the pool
            self.table = torch.randperm(n_pages, generator=g).view(w.batch, max_pages).to(torch.int32).to(dev)
        elif fmt == "delegated":
            W, F = delegated_window()
            self.L = tq.tq_cache_layout_delegated(w.batch, *shape, W, F)
            self.l1 = tq.tq_cache_layout_delegated(1, *shape, W, F)
        else:
            kfmt = tq.TQ_K_INT4 if fmt == "int4" else tq.TQ_K_FP16
            self.L = tq.tq_cache_layout_kv(w.batch, *shape, kfmt)
            self.l1 = tq.tq_cache_layout_kv(1, *shape, kfmt)
        self.kc, self.ks, self.vc, self.vs = tq.alloc_cache(self.L, dev)
        self.tail = tq.alloc_tail(self.L, dev) if fmt == "delegated" else None
        self.wsp = tq.alloc_workspace(self.L, dev)

    def nbytes(self):
        L = self.L
        return int(L.k_bytes + L.codes_bytes + L.scales_bytes * (2 if self.fmt == "int4" else 1) + L.tail_bytes)

    def append_seq(self, b, k, v, n, zero, status, stream):
        """Prefill of sequence b alone (n tokens at position 0) through a batch-1 view."""
        L, tq = self.L, self.tq
        if self.page:
            tq.tq_quantize_append_paged(self.l1, k, v, n, zero, self.table[b:b + 1], self.kc, self.ks, self.vc,
                                        self.vs, status, stream, lambda_k=self.lk, lambda_v=self.lv)
            return
        cs, ss, kst = int(L.code_stride_seq), int(L.scale_stride_seq), int(L.k_stride_seq)
        kc, vc, vs = self.kc[b * kst:(b + 1) * kst], self.vc[b * cs:(b + 1) * cs], self.vs[b * ss:]
        if self.fmt == "delegated":
            ts = int(L.tail_stride_seq) // 2
            tq.tq_append_delegated(self.l1, k, v, n, zero, kc, vc, vs, self.tail[b * ts:(b + 1) * ts], status,
                                   stream)
        else:
            tq.tq_quantize_append(self.l1, k, v, n, zero, kc, None if self.ks is None else self.ks[b * ss:], vc, vs,
                                  status, stream, lambda_k=self.lk, lambda_v=self.lv)

    def append(self, k, v, n, start, status, stream):
        if self.page:
            self.tq.tq_quantize_append_paged(self.L, k, v, n, start, self.table, self.kc, self.ks, self.vc, self.vs,
                                             status, stream, lambda_k=self.lk, lambda_v=self.lv)
        elif self.fmt == "delegated":
            self.tq.tq_append_delegated(self.L, k, v, n, start, self.kc, self.vc, self.vs, self.tail, status, stream)
        else:
            self.tq.tq_quantize_append(self.L, k, v, n, start, self.kc, self.ks, self.vc, self.vs, status, stream,
                                       lambda_k=self.lk, lambda_v=self.lv)

    def decode(self, q, lens, scale, out, status, stream, after_split_event=None):
        if self.page:
            self.tq.tq_decode_attention_paged(self.L, q, lens, self.table, self.kc, self.ks, self.vc, self.vs, scale,
                                              out, self.wsp, status, stream, after_split_event=after_split_event,
                                              lambda_k=self.lk, lambda_v=self.lv, sparse_v_threshold=self.tau)
        elif self.fmt == "delegated":
            self.tq.tq_decode_attention_delegated(self.L, q, lens, self.kc, self.vc, self.vs, self.tail, scale, out,
                                                  self.wsp, status, stream, after_split_event=after_split_event,
                                                  sparse_v_threshold=self.tau)
        else:
            self.tq.tq_decode_attention(self.L, q, lens, self.kc, self.ks, self.vc, self.vs, scale, out, self.wsp,
                                        status, stream, after_split_event=after_split_event, lambda_k=self.lk,
                                        lambda_v=self.lv, sparse_v_threshold=self.tau)


# ----------------------------------------------------------------------------- per-configuration sweep

def _pct(xs, q):
    xs = sorted(xs)
    k = (len(xs) - 1) * q
    lo, hi = int(k), min(int(k) + 1, len(xs) - 1)
    return xs[lo] + (xs[hi] - xs[lo]) * (k - lo)


def _time_graph_pairs(launch, flush, stream, n=10, reps=9):
    """Device time (ms) per call of launch(stream), L2 flushed before each call (flush given)
    or back to back (flush None), finer than one event pair allows (event timestamps on this
    part tick in about 2 us): a CUDA graph of n (flush, call) pairs and one of the n flushes
    alone are replayed in turn between events; per call = (pairs - flushes) / n."""
    import torch
    ga = torch.cuda.CUDAGraph()
    with torch.cuda.graph(ga):
        for _ in range(n):
            if flush is not None:
                flush.add_(1)
            launch(torch.cuda.current_stream())
    gb = None
    if flush is not None:
        gb = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gb):
            for _ in range(n):
                flush.add_(1)
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps + 1):
        pair = []
        for g in (ga, gb):
            if g is None:
                pair.append(0.0)
                continue
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            g.replay()
            b.record(stream)
            torch.cuda.synchronize()
            pair.append(a.elapsed_time(b))
        ts.append((pair[0] - pair[1]) / n)
    ts = ts[1:]  # the first replay of each graph uploads it
    del ga, gb
    return {"median": round(statistics.median(ts), 4), "p10": round(_pct(ts, 0.1), 4),
            "p90": round(_pct(ts, 0.9), 4), "reps": reps, "calls_per_rep": n,
            "method": "graph of (L2 flush, call) pairs minus a graph of the flushes" if flush is not None
            else "graph of back-to-back calls"}


def run_sweep(args):
    """Every workload shape: decode, append and prefill-quantise times, one JSON line per configuration."""
    import torch
    import torch.nn.functional as F
    from compressed_domain_attention_b200 import synthetic as syn
    from compressed_domain_attention_b200 import tq
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    flush = torch.zeros(64 << 20, dtype=torch.float32, device=dev)  # 256 MB > 126 MB L2
    peak, peak_kind = load_peaks()
    cfgs = [("c0", syn.tiny_single_head, False), ("c1", syn.llama3_8b_layer, False)]
    cfgs += [("c2", (lambda T=T: syn.gemma3_1b_sweep(T)), False) for T in (256, 512, 1024, 2048, 4096)]
    cfgs += [("c3", syn.llama31_70b_long, False), ("c4", syn.ragged_serving, False)]
    # the asymmetric (binary16 K, int4 V) and delegated caches on the head_dim-128 shapes
    for fmt in ("fp16", "delegated"):
        cfgs += [("c1", syn.llama3_8b_layer, fmt), ("c3", syn.llama31_70b_long, fmt),
                 ("c4", syn.ragged_serving, fmt)]
    # paged storage (64-token pages) on the long-context and serving shapes
    cfgs += [("c3", syn.llama31_70b_long, "int4/paged64"), ("c4", syn.ragged_serving, "int4/paged64")]
    for tag, make, fmt in cfgs:
        fmt = fmt or "int4"
        page = int(fmt.split("/paged")[1]) if "/paged" in fmt else 0
        fmt = fmt.split("/")[0]
        w = make()
        t = syn.generate(w, device="cuda")
        n_app = max(w.n_append, 1)
        cap = max(w.seq_lens) + n_app
        cache = DeviceCache(w, cap, fmt, dev, page=page)
        status = torch.zeros(1, dtype=torch.int32, device=dev)
        zero = torch.zeros(1, dtype=torch.int32, device=dev)
        kb = [t.k[b][None].contiguous() for b in range(w.batch)]
        vb = [t.v[b][None].contiguous() for b in range(w.batch)]

        def prefill(s=stream):
            for b in range(w.batch):
                cache.append_seq(b, kb[b], vb[b], w.seq_lens[b], zero, status, s)

        prefill()
        pre = _time_graph_pairs(prefill, flush, stream, n=3, reps=5)
        vecs = 2 * sum(w.seq_lens) * w.n_kv_heads
        lens = torch.tensor(w.seq_lens, dtype=torch.int32, device=dev)
        q = t.q.contiguous()
        out = torch.empty((w.batch, w.n_q_heads, w.head_dim), dtype=torch.float32, device=dev)

        def decode():
            cache.decode(q, lens, w.scale, out, status, stream)

        for _ in range(10):
            decode()
        # every timed arm replays CUDA graphs (the dense SDPA below too), so that no host
        # launch work sits between the events
        dec = lambda s: cache.decode(q, lens, w.scale, out, status, s)  # noqa: E731
        cold = _time_graph_pairs(dec, flush, stream)
        nbytes = decode_bytes(w, w.seq_lens, fmt)
        warm = _time_graph_pairs(dec, None, stream) if nbytes < 64e6 else None
        kn, vn = t.k_new.contiguous() if w.n_append else None, t.v_new.contiguous() if w.n_append else None
        app = None
        if w.n_append:
            app = _time_graph_pairs(lambda s: cache.append(kn, vn, w.n_append, lens, status, s), flush, stream)
        dense = None
        if w.dtype != torch.float32:
            ks_d = [t.k[b].permute(1, 0, 2).contiguous()[None] for b in range(w.batch)]
            vs_d = [t.v[b].permute(1, 0, 2).contiguous()[None] for b in range(w.batch)]
            qd = q.view(w.batch, w.n_q_heads, 1, w.head_dim)

            def dense_fn():
                for b in range(w.batch):
                    F.scaled_dot_product_attention(qd[b:b + 1], ks_d[b], vs_d[b], scale=w.scale, enable_gqa=True)

            dense_fn()
            dense = _time_graph_pairs(lambda s: dense_fn(), flush, stream)
            del ks_d, vs_d
        torch.cuda.synchronize()
        if int(status.item()) != 0:
            raise RuntimeError(f"device status {int(status.item())} in the sweep ({w.name})")
        ms = cold["median"]
        line = {"sweep": tag, "workload": w.name, "k_format": fmt, "page_tokens": page, "batch": w.batch,
                "tokens": sum(w.seq_lens), "cache_bytes_read": nbytes,
                "decode_ms_cold_l2": cold, "decode_gbs": round(nbytes / ms / 1e6, 1),
                "pct_of_8_tbs": round(nbytes / ms / 1e6 / 80.0, 2),
                "pct_of_measured_hbm": round(nbytes / ms / 1e6 / peak * 100.0, 2), "peak_kind": peak_kind,
                "decode_steps_per_s": round(w.batch / ms * 1e3, 1),
                "kv_tokens_per_s": round(sum(w.seq_lens) / ms * 1e3, 1),
                "decode_ms_warm_l2": warm,
                "prefill_quantize": {"vectors": vecs, "launches": w.batch, "ms": pre,
                                     "vectors_per_s": round(vecs / pre["median"] * 1e3, 1)},
                "append_ms_cold_l2": app,
                "bf16_dense_sdpa_ms_cold_l2": dense,
                "speedup_vs_bf16_dense": round(dense["median"] / ms, 2) if dense else None}
        print(json.dumps(line), flush=True)
        del cache, t, kb, vb
        torch.cuda.empty_cache()
    return 0

# ----------------------------------------------------------------------------- main paths

def run_reference(args):
    """--impl reference: the CPU oracle on the host cores, bounded sample per step (rank 0 only)."""
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    from compressed_domain_attention_b200 import synthetic as syn
    w = get_workload(args.workload)
    if w.n_append == 0:
        w.n_append = 1
    seqs = oracle_sample(w, 8192)
    t = syn.generate(w, device="cpu", seq_subset=seqs)
    o = OracleStep(w, t, seqs, getattr(args, "k_format", "int4"), getattr(args, "lam", False),
                   getattr(args, "sparse_v", 0.0))
    for _ in range(args.warmup):
        o.run()
    tot_t = sum(o.run() for _ in range(args.steps))
    value = o.nbytes * args.steps / tot_t / 1e9
    sample = (f"each step: append + decode on {len(seqs)} of {w.batch} sequences "
              f"({o.ntok} KV tokens x {w.n_q_heads} q heads), single-threaded C++ oracle")
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(tot_t / args.steps * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32 encode / f64 attention",
            "data": "synthetic (seeded)", "config": {"workload": w.name, "global_batch": w.batch,
                                                     "k_format": getattr(args, "k_format", "int4"),
                                                     "lambda": bool(getattr(args, "lam", False)),
                                                     "sparse_v_threshold": getattr(args, "sparse_v", 0.0)},
            "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample,
                             "cpu_model": cpu_model(), "host_cores": host_cores()},
            "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)
    return 0


class StepTiming:
    """Device state and timings of one workload's step (append one token per sequence + decode)."""


def time_device_steps(w, fmt, args, dev, stream, rank, local):
    """Prefill the workload's cache (untimed), then time K steps of (append, decode).

    The K timed steps are captured once as a CUDA graph and replayed between CUDA
    events, bracketed by a barrier and a synchronize; a second pass of the same K
    steps records an event between the split-K and merge kernels for per-kernel
    durations. Clocks are sampled with nvidia-smi during the graph-timed region.
    """
    import torch
    from compressed_domain_attention_b200 import synthetic as syn
    r = StepTiming()
    if w.n_append == 0:
        w.n_append = 1
    cap = max(w.seq_lens) + w.n_append
    t = syn.generate(w, device="cuda")
    cache = DeviceCache(w, cap, fmt, dev, args.lam, args.sparse_v, args.paged)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    zero = torch.zeros(1, dtype=torch.int32, device=dev)
    for b in range(w.batch):
        cache.append_seq(b, t.k[b][None].contiguous(), t.v[b][None].contiguous(), w.seq_lens[b], zero, status,
                         stream)
    torch.cuda.synchronize()
    r.prefill = None
    if w.batch == 1 and fmt != "delegated" and rank == 0:
        # the one-sequence prefill again (same data, same rows), device-timed with L2 flushed before
        # each call: the append kernel on a long prompt
        flush = torch.zeros(64 << 20, dtype=torch.float32, device=dev)
        kp, vp = t.k[0][None].contiguous(), t.v[0][None].contiguous()
        r.prefill = _time_graph_pairs(lambda s: cache.append_seq(0, kp, vp, w.seq_lens[0], zero, status, s),
                                      flush, stream, n=3, reps=5)
        del flush, kp, vp
        torch.cuda.synchronize()
    lens = torch.tensor(w.seq_lens, dtype=torch.int32, device=dev)
    lens1 = lens + w.n_append
    q = t.q.contiguous()
    k_new, v_new = t.k_new.contiguous(), t.v_new.contiguous()
    out = torch.empty((w.batch, w.n_q_heads, w.head_dim), dtype=torch.float32, device=dev)

    n_ev = args.steps
    ev_a = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
    ev_s = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
    ev_b = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]

    # One step appends each sequence's new token at its prefix length and decodes over
    # prefix + 1, so every step repeats the same work (with the delegated cache, the
    # same fold of the tail into the int4 body where a sequence's length crosses a
    # fold boundary).
    def step(i=None):
        cache.append(k_new, v_new, w.n_append, lens, status, stream)
        if i is not None:
            ev_a[i].record(stream)
            cache.decode(q, lens1, w.scale, out, status, stream, after_split_event=ev_s[i])
            ev_b[i].record(stream)
        else:
            cache.decode(q, lens1, w.scale, out, status, stream)

    for _ in range(max(args.warmup, 3)):
        step()
    for e in ev_s:  # torch creates the CUDA event on first record; the library re-records it later
        e.record(stream)
    torch.cuda.synchronize()
    barrier(dev)
    clocks = ClockSampler(local) if (rank == 0 and not args.no_clocks) else None
    if clocks:
        clocks.start()
        time.sleep(0.3)
    torch.cuda.synchronize()
    # The K steps captured once as a CUDA graph, so that the timed region measures the
    # device (a ~50 us step is otherwise paced by the host's launch calls); eager
    # launches if capture is refused.
    step_mode = "cuda graph of the K steps"
    sgraph = torch.cuda.CUDAGraph()
    sstream = torch.cuda.Stream(device=dev)
    try:
        sstream.wait_stream(stream)
        with torch.cuda.graph(sgraph, stream=sstream):
            for _ in range(args.steps):
                cache.append(k_new, v_new, w.n_append, lens, status, sstream)
                cache.decode(q, lens1, w.scale, out, status, sstream)
        with torch.cuda.stream(sstream):
            sgraph.replay()
        torch.cuda.synchronize()
    except Exception as exc:  # noqa: BLE001 - reported in the output line
        sgraph = None
        step_mode = f"eager launches (graph capture failed: {type(exc).__name__})"
        torch.cuda.synchronize()
    barrier(dev)
    # timed region: the production path (append, split-K and merge kernels back to back)
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if sgraph is not None:
        sstream.wait_stream(stream)
        with torch.cuda.stream(sstream):  # replay() launches on the current stream
            start.record(sstream)
            sgraph.replay()
            stop.record(sstream)
    else:
        start.record(stream)
        for _ in range(args.steps):
            step()
        stop.record(stream)
    torch.cuda.synchronize()
    barrier(dev)
    r.clocks = clocks.stop() if clocks else None
    r.elapsed = start.elapsed_time(stop) / 1e3
    del sgraph
    # second timed pass of the same steps with an event between the split-K and
    # merge kernels: per-kernel durations for the roofline. Eager launches: a short
    # GPU spin first lets the host queue the steps ahead of the device, so no host
    # gap (tensor-map encoding, launch calls) falls between an event and its kernel.
    torch.cuda._sleep(int(2e6))
    for i in range(args.steps):
        step(i)
    torch.cuda.synchronize()
    r.split_ms = [ev_a[i].elapsed_time(ev_s[i]) for i in range(args.steps)]
    r.merge_ms = [ev_s[i].elapsed_time(ev_b[i]) for i in range(args.steps)]
    st = int(status.item())
    if st != 0:
        raise RuntimeError(f"device status {st} during the benchmark ({w.name})")
    r.w, r.t, r.cache, r.status = w, t, cache, status
    r.lens, r.lens1, r.q, r.k_new, r.v_new, r.out = lens, lens1, q, k_new, v_new, out
    r.step, r.step_mode = step, step_mode
    r.lens_step = [x + w.n_append for x in w.seq_lens]
    r.bytes_split = split_bytes(w, r.lens_step, fmt)
    r.bytes_step = decode_bytes(w, r.lens_step, fmt) + append_bytes(w, 2 if w.dtype != torch.float32 else 4, fmt)
    return r


def traffic_key(w, fmt, paged):
    return (f"decode_split_kernel/{w.name}" + {"int4": "", "fp16": "/k_fp16", "delegated": "/delegated"}[fmt]
            + (f"/paged{paged}" if paged else ""))


def roofline_record(r, fmt, paged, dev):
    """Roofline of the split-K kernel: algorithmic bytes per launch / event-timed launch duration."""
    peak, peak_kind = load_peaks()
    split_avg = max_over_ranks(statistics.mean(r.split_ms), dev)
    merge_avg = max_over_ranks(statistics.mean(r.merge_ms), dev)
    achieved = r.bytes_split / (split_avg / 1e3) / 1e9
    return {"bound": "hbm", "kernel": "decode_split_kernel", "achieved": round(achieved, 1),
            "peak": peak, "unit": "GB/s", "frac": round(achieved / peak, 4),
            "traffic": load_traffic(traffic_key(r.w, fmt, paged)),
            "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured"
            else "fallback 6.65 TB/s",
            "algorithmic_bytes_per_launch": r.bytes_split, "avg_launch_ms": round(split_avg, 4),
            "merge_avg_ms": round(merge_avg, 4)}


def long_context_record(args, fmt, dev, stream, rank, local, ws):
    """The 131072-token Llama-3.1-70B-shaped step (64 q / 8 kv heads), timed like the headline, and its
    131072-token prefill (the append kernel on a long prompt)."""
    import torch
    from compressed_domain_attention_b200 import synthetic as syn
    w = syn.llama31_70b_long()
    r = time_device_steps(w, fmt, args, dev, stream, rank, local)
    max_t = max_over_ranks(r.elapsed, dev)
    peak, _ = load_peaks()
    rec = {"workload": w.name, "n_q_heads": w.n_q_heads, "n_kv_heads": w.n_kv_heads, "head_dim": w.head_dim,
           "kv_tokens_per_seq_step": r.lens_step, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": round(max_t / args.steps * 1e3, 4),
           "value": round(ws * r.bytes_step * args.steps / max_t / 1e9, 2), "unit": UNIT,
           "pct_of_measured_hbm": round(100.0 * r.bytes_step * args.steps / max_t / 1e9 / peak, 2),
           "pct_of_8tbs": round(100.0 * r.bytes_step * args.steps / max_t / 1e9 / 8000.0, 2),
           "kv_tokens_per_s": round(ws * sum(r.lens_step) * args.steps / max_t, 1),
           "algorithmic_bytes_per_step": r.bytes_step,
           "roofline": roofline_record(r, fmt, args.paged, dev), "step_launch": r.step_mode,
           "l2": f"inputs larger than L2 (cache {r.cache.nbytes() / 1e9:.2f} GB > 126 MB), no flush"}
    if r.clocks:
        rec["clocks"] = r.clocks
    if r.prefill is not None:
        T = w.seq_lens[0]
        pw = syn.Workload(w.name, 1, w.n_q_heads, w.n_kv_heads, w.head_dim, [0], w.dtype, 0, n_append=T)
        nb = append_bytes(pw, 2 if w.dtype != torch.float32 else 4, fmt)
        ms = r.prefill["median"]
        rec["prefill_quantize"] = {
            "tokens": T, "vectors": 2 * T * w.n_kv_heads, "ms": ms, "timing": r.prefill,
            "algorithmic_bytes": nb, "gb_per_s": round(nb / ms / 1e6, 1),
            "frac_of_measured_hbm": round(nb / ms / 1e6 / peak, 4),
            "kernel": "quantize_rows_kernel" if w.head_dim in (64, 128) else "quantize_append_kernel",
            "l2": "flushed before each call"}
    return rec


def run_tq(args):
    import torch
    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_dist("nccl")
    w = get_workload(args.workload)
    fmt = args.k_format
    if args.lam and fmt == "delegated":
        raise SystemExit("--lambda applies to the int4 and fp16 formats (the delegated tail is binary16)")
    if args.paged and fmt == "delegated":
        raise SystemExit("--paged applies to the int4 and fp16 formats")
    stream = torch.cuda.current_stream()
    r = time_device_steps(w, fmt, args, dev, stream, rank, local)
    cache, L, status, out, q, k_new, v_new = r.cache, r.cache.L, r.status, r.out, r.q, r.k_new, r.v_new
    lens, lens1, t, elapsed = r.lens, r.lens1, r.t, r.elapsed

    # e2e: host buffers in pinned memory, every step's copies inside the timed region.
    # As a serving loop would run it: a copy stream brings step i+1's inputs in and
    # step i's output back while the compute stream runs step i (double-buffered
    # device inputs and outputs, ordered by events).
    h_k = [k_new.cpu().pin_memory() for _ in range(2)]
    h_v = [v_new.cpu().pin_memory() for _ in range(2)]
    h_q = [q.cpu().pin_memory() for _ in range(2)]
    h_out = [torch.empty_like(out, device="cpu").pin_memory() for _ in range(2)]
    d_k = [torch.empty_like(k_new) for _ in range(2)]
    d_v = [torch.empty_like(v_new) for _ in range(2)]
    d_q = [torch.empty_like(q) for _ in range(2)]
    d_out = [torch.empty_like(out) for _ in range(2)]
    cstream = torch.cuda.Stream(device=dev)
    gstream = torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]     # inputs of the buffer landed
    ev_done = [torch.cuda.Event() for _ in range(2)]   # compute on the buffer finished
    ev_out = [torch.cuda.Event() for _ in range(2)]    # output of the buffer copied back

    def e2e_loop(n, cs):
        """n steps on compute stream cs; copies on cstream (forked from and joined back to cs)."""
        cstream.wait_stream(cs)

        def h2d(i):
            j = i % 2
            with torch.cuda.stream(cstream):
                if i >= 2:
                    cstream.wait_event(ev_done[j])  # step i-2 no longer reads these inputs
                d_k[j].copy_(h_k[j], non_blocking=True)
                d_v[j].copy_(h_v[j], non_blocking=True)
                d_q[j].copy_(h_q[j], non_blocking=True)
                ev_in[j].record(cstream)

        h2d(0)
        for i in range(n):
            j = i % 2
            if i + 1 < n:
                h2d(i + 1)
            cs.wait_event(ev_in[j])
            if i >= 2:
                cs.wait_event(ev_out[j])  # step i-2's output was copied out of d_out[j]
            cache.append(d_k[j], d_v[j], w.n_append, lens, status, cs)
            cache.decode(d_q[j], lens1, w.scale, d_out[j], status, cs)
            ev_done[j].record(cs)
            with torch.cuda.stream(cstream):
                cstream.wait_event(ev_done[j])
                h_out[j].copy_(d_out[j], non_blocking=True)
                ev_out[j].record(cstream)
        cs.wait_stream(cstream)

    e2e_loop(3, stream)
    torch.cuda.synchronize()
    # The K steps (copies, append, decode) captured once as a CUDA graph, as a
    # fixed-shape serving step would run; eager launches if capture is refused.
    e2e_mode = "cuda graph of the K steps"
    graph = torch.cuda.CUDAGraph()
    try:
        gstream.wait_stream(stream)
        with torch.cuda.graph(graph, stream=gstream):
            e2e_loop(args.steps, gstream)
        with torch.cuda.stream(gstream):
            graph.replay()
        torch.cuda.synchronize()
    except Exception as exc:  # noqa: BLE001 - reported in the output line
        graph = None
        e2e_mode = f"eager launches (graph capture failed: {type(exc).__name__})"
        torch.cuda.synchronize()
    barrier(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if graph is not None:
        gstream.wait_stream(stream)
        with torch.cuda.stream(gstream):  # replay() launches on the current stream
            e0.record(gstream)
            graph.replay()
            e1.record(gstream)
    else:
        e0.record(stream)
        e2e_loop(args.steps, stream)
        e1.record(stream)
    torch.cuda.synchronize()
    barrier(dev)
    e2e_s = e0.elapsed_time(e1) / 1e3
    if not torch.equal(h_out[(args.steps - 1) % 2], out.cpu()):
        raise RuntimeError("end-to-end output differs from the device-timed output")
    del graph

    refs = {} if args.no_references else reference_points(w, t, L, cache.kc, cache.ks, cache.vc, cache.vs, lens1,
                                                          q, dev, stream, args, fmt=fmt)

    lens_step = r.lens_step
    bytes_step = r.bytes_step
    max_t = max_over_ranks(elapsed, dev)
    max_e2e = max_over_ranks(e2e_s, dev)
    peak, _ = load_peaks()
    cache_bytes = cache.nbytes()
    extra = {
        "tokens_per_s": round(ws * w.batch * w.n_append * args.steps / max_t, 1),
        "kv_tokens_per_s": round(ws * sum(lens_step) * args.steps / max_t, 1),
        "pct_of_measured_hbm": round(100.0 * bytes_step / max_t * args.steps / 1e9 / peak, 2),
        "pct_of_8tbs": round(100.0 * bytes_step / max_t * args.steps / 1e9 / 8000.0, 2),
        "roofline": roofline_record(r, fmt, args.paged, dev),
        "e2e": {"value": round(ws * bytes_step * args.steps / max_e2e / 1e9, 2), "unit": UNIT,
                "h2d_bytes_per_step": int(k_new.numel() * k_new.element_size() * 2 + q.numel() * q.element_size()),
                "d2h_bytes_per_step": int(out.numel() * out.element_size()),
                "copies": "pinned host buffers; step i+1's inputs in and step i's output out on a copy "
                          "stream while step i computes (double-buffered, event-ordered)", "launch": e2e_mode},
        "gpu_launches": (4 if fmt == "delegated" else 3) * args.steps,
        "step_launch": r.step_mode,
        "kernel_timing": "split-K/merge durations from a second pass of the same K steps with an event "
                         "between the two kernels (the timed region itself launches the merge as a "
                         "programmatic dependent)",
    }
    if r.clocks:
        extra["clocks"] = r.clocks
    extra.update(refs)
    cfg = {"workload": w.name, "global_batch": w.batch * ws, "kv_tokens_per_seq_step": lens_step if w.batch <= 4
           else {"min": min(lens_step), "max": max(lens_step), "sum": sum(lens_step)},
           "n_q_heads": w.n_q_heads, "n_kv_heads": w.n_kv_heads, "head_dim": w.head_dim,
           "k_format": args.k_format, "lambda": bool(args.lam), "sparse_v_threshold": args.sparse_v,
           "page_tokens": args.paged,
           "parallelism": f"replicas x{ws}" if ws > 1 else "single GPU",
           "l2": f"inputs larger than L2 (cache {cache_bytes / 1e9:.2f} GB per replica > 126 MB), no flush",
           "algorithmic_bytes_per_step": bytes_step}
    total_bytes = sum_over_ranks(bytes_step * args.steps, dev)  # every rank takes part
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        extra["cpu_baseline"] = cpu_baseline(w, t, 300000, fmt, args.lam, args.sparse_v)
    # the long-context workload (131072 tokens, query groups of 8) as a sub-record of the same line
    if not args.no_long_context and args.workload != "llama31_70b_long":
        del r, cache, t, h_k, h_v, h_q, h_out, d_k, d_v, d_q, d_out
        torch.cuda.empty_cache()
        extra["long_context"] = long_context_record(args, fmt, dev, stream, rank, local, ws)
    if rank == 0:
        line = assemble_line(n_gpus=ws, steps=args.steps, warmup=args.warmup, total_bytes_all_ranks=total_bytes,
                             max_time_s=max_t, workload=cfg, extra=extra)
        print(json.dumps(line), flush=True)
    import torch.distributed as dist
    if dist.is_initialized():
        dist.destroy_process_group()
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    if args.sweep:
        return run_sweep(args)
    return run_tq(args)


if __name__ == "__main__":
    sys.exit(main())
