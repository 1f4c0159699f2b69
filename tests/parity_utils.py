"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI
and the CPU oracle on the same seeded inputs, and compare."""
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

import oracle
from compressed_domain_attention_b200 import tq

ATOL = 2e-3     # decode tolerance: max-abs error vs the oracle's fp32 result
RTOL_L2 = 1e-3  # and relative L2 error


def parallel_map(fn, items):
    """fn(item) for every item on a host thread pool. The oracle is reached through ctypes,
    whose foreign calls release the interpreter lock, so independent sequences or heads
    run on separate cores; each call is the unchanged single-threaded oracle."""
    items = list(items)
    n = max(1, min(len(items), os.cpu_count() or 1))
    with ThreadPoolExecutor(max_workers=n) as ex:
        return list(ex.map(fn, items))


def oracle_decode_all(decode_fn, batch, n_q, heads_per_task=None):
    """Every (sequence, q head) of an oracle decode, split into independent tasks.

    decode_fn(which) -> (out [B][Hq][D], status) computes the rows selected by the
    uint8 mask which [B][Hq]; tasks are whole sequences (or groups of heads of one
    sequence when heads_per_task is given) and their rows are gathered into one
    output. Returns (out, OR of the statuses)."""
    hp = heads_per_task or n_q
    tasks = [(b, h0) for b in range(batch) for h0 in range(0, n_q, hp)]

    def one(task):
        b, h0 = task
        which = np.zeros((batch, n_q), np.uint8)
        which[b, h0:h0 + hp] = 1
        out, st = decode_fn(which)
        return task, out[b, h0:h0 + hp].copy(), st

    full = None
    status = 0
    for (b, h0), rows, st in parallel_map(one, tasks):
        if full is None:
            full = np.zeros((batch, n_q, rows.shape[-1]), np.float32)
        full[b, h0:h0 + hp] = rows
        status |= st
    return full, status


def np_f32(t):
    if isinstance(t, np.ndarray):
        return np.ascontiguousarray(t, np.float32)
    return t.detach().to("cpu", torch.float32).contiguous().numpy()


class GpuCache:
    """A packed K/V cache in device memory laid out by tq_cache_layout."""

    def __init__(self, batch, max_seq, n_kv, n_q, D, sign_seed=0, device="cuda", k_format=tq.TQ_K_INT4):
        self.layout = tq.tq_cache_layout_kv(batch, max_seq, n_kv, n_q, D, k_format, 32, sign_seed)
        self.k_codes, self.k_scales, self.v_codes, self.v_scales = tq.alloc_cache(self.layout, device)
        self.device = device
        self.kf16 = k_format == tq.TQ_K_FP16

    def seq_view(self, b):
        """(layout, k_codes, k_scales, v_codes, v_scales) for sequence b alone (a batch-1 view)."""
        L = self.layout
        l1 = tq.tq_cache_layout_kv(1, L.max_seq, L.n_kv_heads, L.n_q_heads, L.head_dim, L.k_format, 32, L.sign_seed)
        cs, ss, ks_ = int(L.code_stride_seq), int(L.scale_stride_seq), int(L.k_stride_seq)
        return (l1, self.k_codes[b * ks_:(b + 1) * ks_], None if self.kf16 else self.k_scales[b * ss:],
                self.v_codes[b * cs:(b + 1) * cs], self.v_scales[b * ss:])

    def append_seq(self, b, k, v, start, status=None):
        """Append k, v [n][Hkv][D] to sequence b at position start."""
        l1, kc, ks, vc, vs = self.seq_view(b)
        sp = torch.tensor([start], dtype=torch.int32, device=self.device)
        tq.tq_quantize_append(l1, k[None].contiguous(), v[None].contiguous(), k.shape[0], sp, kc, ks, vc, vs, status)

    def append_all(self, k, v, start_pos, status=None):
        """k, v [B][n][Hkv][D]; start_pos int list."""
        sp = torch.tensor(start_pos, dtype=torch.int32, device=self.device)
        tq.tq_quantize_append(self.layout, k.contiguous(), v.contiguous(), k.shape[1], sp, self.k_codes,
                              self.k_scales, self.v_codes, self.v_scales, status)

    def host_arrays(self):
        """(k_codes, k_scales, v_codes, v_scales) as numpy [B][S][Hkv][...] (scales as uint16 bits)."""
        L = self.layout
        B, S, H, D = L.batch, L.max_seq, L.n_kv_heads, L.head_dim
        n_s = B * S * H * (D // 32)
        vc = self.v_codes.cpu().numpy().reshape(B, S, H, D // 2)
        if self.kf16:  # binary16 K bits [B][S][H][D], no K scales
            kc = self.k_codes.cpu().numpy().view(np.uint16).reshape(B, S, H, D)
            ks = None
        else:
            kc = self.k_codes.cpu().numpy().reshape(B, S, H, D // 2)
            ks = self.k_scales[:n_s].cpu().numpy().view(np.uint16).reshape(B, S, H, D // 32)
        vs = self.v_scales[:n_s].cpu().numpy().view(np.uint16).reshape(B, S, H, D // 32)
        return kc, ks, vc, vs

    def decode(self, q, seq_lens, sm_scale, status=None, **opts):
        L = self.layout
        out = torch.full((L.batch, L.n_q_heads, L.head_dim), float("nan"), dtype=torch.float32, device=self.device)
        ws = tq.alloc_workspace(L, self.device)
        lens = torch.tensor(seq_lens, dtype=torch.int32, device=self.device)
        tq.tq_decode_attention(L, q.contiguous(), lens, self.k_codes, self.k_scales, self.v_codes, self.v_scales,
                               sm_scale, out, ws, status, **opts)
        return out


class OracleCache:
    def __init__(self, batch, max_seq, n_kv, D, sign_seed=0, kf16=False):
        self.signs = oracle.sign_vector(sign_seed, D)
        self.kf16 = kf16
        if kf16:
            self.kc, self.ks = oracle.new_k16_cache(batch, max_seq, n_kv, D), None
        else:
            self.kc, self.ks = oracle.new_cache(batch, max_seq, n_kv, D)
        self.vc, self.vs = oracle.new_cache(batch, max_seq, n_kv, D)

    def append_seq(self, b, k, v, start):
        sp = np.array([start], np.int32)
        if self.kf16:
            st = oracle.quantize_append_kf16(self.signs, np_f32(k)[None], np_f32(v)[None], sp, self.kc[b:b + 1],
                                             self.vc[b:b + 1], self.vs[b:b + 1])
        else:
            st = oracle.quantize_append(self.signs, np_f32(k)[None], np_f32(v)[None], sp, self.kc[b:b + 1],
                                        self.ks[b:b + 1], self.vc[b:b + 1], self.vs[b:b + 1])
        assert st == 0

    def append_seqs(self, t, seqs):
        """Prefill the listed sequences of tensors t (each at position 0) on a thread pool."""
        parallel_map(lambda b: self.append_seq(b, t.k[b], t.v[b], 0), [b for b in seqs if t.k[b] is not None
                                                                         and t.k[b].shape[0] > 0])

    def decode_all(self, q, seq_lens, sm_scale, heads_per_task=None):
        """Every (sequence, head) of the decode, on a thread pool. -> (out, status)."""
        qn = np_f32(q)
        return oracle_decode_all(lambda which: self.decode(qn, seq_lens, sm_scale, which), qn.shape[0],
                                 qn.shape[1], heads_per_task)

    def decode(self, q, seq_lens, sm_scale, which=None):
        lens = np.asarray(seq_lens, np.int32)
        if self.kf16:
            return oracle.decode_attention_kf16(self.signs, np_f32(q), lens, self.kc, self.vc, self.vs, sm_scale,
                                                which)
        out, st = oracle.decode_attention(self.signs, np_f32(q), lens, self.kc, self.ks, self.vc, self.vs, sm_scale,
                                          which)
        return out, st


class DelegatedGpuCache:
    """A delegated hot/cold cache in device memory (binary16 K, binary16 V tail + int4 V body)."""

    def __init__(self, batch, max_seq, n_kv, n_q, D, window, fold, sign_seed=0, device="cuda"):
        self.layout = tq.tq_cache_layout_delegated(batch, max_seq, n_kv, n_q, D, window, fold, 32, sign_seed)
        self.k16, _, self.v_codes, self.v_scales = tq.alloc_cache(self.layout, device)
        self.tail = tq.alloc_tail(self.layout, device)
        self.device = device
        self.window, self.fold = window, fold

    def seq_view(self, b):
        L = self.layout
        l1 = tq.tq_cache_layout_delegated(1, L.max_seq, L.n_kv_heads, L.n_q_heads, L.head_dim, self.window,
                                          self.fold, 32, L.sign_seed)
        cs, ss, ks_ = int(L.code_stride_seq), int(L.scale_stride_seq), int(L.k_stride_seq)
        ts = int(L.tail_stride_seq) // 2
        return (l1, self.k16[b * ks_:(b + 1) * ks_], self.v_codes[b * cs:(b + 1) * cs], self.v_scales[b * ss:],
                self.tail[b * ts:(b + 1) * ts])

    def append_seq(self, b, k, v, start, status=None):
        l1, kc, vc, vs, tl = self.seq_view(b)
        sp = torch.tensor([start], dtype=torch.int32, device=self.device)
        tq.tq_append_delegated(l1, k[None].contiguous(), v[None].contiguous(), k.shape[0], sp, kc, vc, vs, tl, status)

    def append_all(self, k, v, start_pos, status=None):
        sp = torch.tensor(start_pos, dtype=torch.int32, device=self.device)
        tq.tq_append_delegated(self.layout, k.contiguous(), v.contiguous(), k.shape[1], sp, self.k16, self.v_codes,
                               self.v_scales, self.tail, status)

    def host_arrays(self):
        """(k16 bits [B][S][H][D], v_codes, v_scales bits, tail bits [B][W][H][D]) as numpy."""
        L = self.layout
        B, S, H, D = L.batch, L.max_seq, L.n_kv_heads, L.head_dim
        n_s = B * S * H * (D // 32)
        k16 = self.k16.cpu().numpy().view(np.uint16).reshape(B, S, H, D)
        vc = self.v_codes.cpu().numpy().reshape(B, S, H, D // 2)
        vs = self.v_scales[:n_s].cpu().numpy().view(np.uint16).reshape(B, S, H, D // 32)
        tail = self.tail.cpu().numpy().view(np.uint16).reshape(B, self.window, H, D)
        return k16, vc, vs, tail

    def decode(self, q, seq_lens, sm_scale, status=None, **opts):
        L = self.layout
        out = torch.full((L.batch, L.n_q_heads, L.head_dim), float("nan"), dtype=torch.float32, device=self.device)
        ws = tq.alloc_workspace(L, self.device)
        lens = torch.tensor(seq_lens, dtype=torch.int32, device=self.device)
        tq.tq_decode_attention_delegated(L, q.contiguous(), lens, self.k16, self.v_codes, self.v_scales, self.tail,
                                         sm_scale, out, ws, status, **opts)
        return out


class DelegatedOracleCache:
    def __init__(self, batch, max_seq, n_kv, D, window, fold, sign_seed=0):
        self.signs = oracle.sign_vector(sign_seed, D)
        self.window, self.fold = window, fold
        self.k16 = oracle.new_k16_cache(batch, max_seq, n_kv, D)
        self.vc, self.vs = oracle.new_cache(batch, max_seq, n_kv, D)
        self.tail = oracle.new_tail(batch, window, n_kv, D)

    def append_seq(self, b, k, v, start):
        st = oracle.append_delegated(self.signs, np_f32(k)[None], np_f32(v)[None], np.array([start], np.int32),
                                     self.window, self.fold, self.k16[b:b + 1], self.vc[b:b + 1],
                                     self.vs[b:b + 1], self.tail[b:b + 1])
        assert st == 0

    def decode_all(self, q, seq_lens, sm_scale, heads_per_task=None):
        qn = np_f32(q)
        return oracle_decode_all(lambda which: self.decode(qn, seq_lens, sm_scale, which), qn.shape[0],
                                 qn.shape[1], heads_per_task)

    def decode(self, q, seq_lens, sm_scale, which=None):
        return oracle.decode_attention_delegated(self.signs, np_f32(q), np.asarray(seq_lens, np.int32), self.k16,
                                                 self.vc, self.vs, self.tail, self.window, self.fold, sm_scale,
                                                 which)


def assert_delegated_caches_equal(gpu, orc, seqs, lens):
    """Bit-exact where the cache is defined: every K row, the int4 body below the cold length,
    and the tail slots of the hot tokens (slots of folded tokens are unspecified)."""
    k16, vc, vs, tail = gpu.host_arrays()
    W, F = gpu.window, gpu.fold
    for b in seqs:
        n = lens[b]
        nc = oracle.cold_length(n, W, F)
        assert np.array_equal(k16[b, :n], orc.k16[b, :n]), f"binary16 K differs in sequence {b}"
        assert np.array_equal(vc[b, :nc], orc.vc[b, :nc]), f"V codes differ in sequence {b}"
        assert np.array_equal(vs[b, :nc], orc.vs[b, :nc]), f"V scales differ in sequence {b}"
        live = [t % W for t in range(nc, n)]
        assert np.array_equal(tail[b, live], orc.tail[b, live]), f"V tail differs in sequence {b}"


def assert_close(got, ref, atol=ATOL, rtol_l2=RTOL_L2, what=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    max_abs = float(err.max()) if err.size else 0.0
    rel = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30))
    assert max_abs <= atol and rel <= rtol_l2, f"{what}: max_abs {max_abs:.3e} (<= {atol}), rel_l2 {rel:.3e} (<= {rtol_l2})"
    return max_abs, rel
