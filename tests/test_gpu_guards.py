"""Guard-byte (canary) checks of every buffer the kernels touch.

compute-sanitizer is not available on this GPU pool, so writes out of bounds are
caught with guards instead: each caller buffer (K and V codes, scales, binary16
K, the delegated cache's V tail, the paged pools, the decode workspace and the
output) sits between two 4 KB guard regions filled with a pattern, and after
appends and decodes the guards must be unchanged.

Reads past the valid rows are checked by their effect: every cache row past a
sequence's length, and the scales' read-ahead padding, hold garbage (binary16
NaN scales, arbitrary code bytes), and the workspace and output start as NaN
patterns. The decode reads scale rows in tile-sized blocks that run past the
last valid token, and paged storage reads an unmapped page's tile through a
tensor copy that starts past the pool; none of those bytes may reach the
output, which must still match the oracle (computed on clean caches).

Cases: ragged lengths at unit, tile and split edges, one sequence filling
max_seq exactly (its last tile's scale read-ahead runs into the padding), both
score layouts (query groups of 4 and 8), binary16 K, the delegated cache and
paged pools with and without an unmapped page.
"""
import numpy as np
import pytest
import torch

import oracle
from compressed_domain_attention_b200 import synthetic as syn
from compressed_domain_attention_b200 import tq
from tests.parity_utils import (DelegatedOracleCache, OracleCache, assert_close, np_f32, oracle_decode_all,
                                parallel_map)

pytestmark = pytest.mark.gpu

GUARD = 4096
GUARD_BYTE = 0xA5


class Guarded:
    """nbytes of device memory between two guard regions; `inner` fills the buffer itself."""

    def __init__(self, nbytes, inner):
        self.n = int(nbytes)
        self.full = torch.full((self.n + 2 * GUARD,), GUARD_BYTE, dtype=torch.uint8, device="cuda")
        self.view = self.full[GUARD:GUARD + self.n]
        self.view.fill_(inner)

    def as16(self):
        return self.view[: self.n // 2 * 2].view(torch.int16)

    def as32f(self):
        return self.view.view(torch.float32)

    def intact(self):
        f = self.full
        return bool((f[:GUARD] == GUARD_BYTE).all().item()) and bool((f[GUARD + self.n:] == GUARD_BYTE).all().item())


def all_intact(bufs):
    torch.cuda.synchronize()
    bad = [name for name, b in bufs.items() if not b.intact()]
    assert not bad, f"guard bytes overwritten next to: {bad}"


def decode_buffers(L, batch, n_q, D):
    ws = Guarded(L.decode_workspace_bytes, 0xFF)      # NaN patterns: the kernels must write what they read
    out = Guarded(batch * n_q * D * 4, 0xFF)
    return ws, out


@pytest.mark.parametrize("G,k_format", [(4, tq.TQ_K_INT4), (8, tq.TQ_K_INT4), (4, tq.TQ_K_FP16),
                                        (8, tq.TQ_K_FP16)])
def test_guards_contiguous_cache(G, k_format):
    max_seq = 1000
    lens = [max_seq, 1, 31, 32, 33, 255, 256, 257, 700]
    B, Hkv, D = len(lens), 8, 128
    w = syn.Workload(f"guards_g{G}", B, Hkv * G, Hkv, D, lens, torch.bfloat16, 71, max_seq=max_seq)
    t = syn.generate(w)
    kf = k_format == tq.TQ_K_FP16
    L = tq.tq_cache_layout_kv(B, max_seq, Hkv, Hkv * G, D, k_format)
    bufs = {"k": Guarded(L.k_bytes, 0x5A), "v_codes": Guarded(L.codes_bytes, 0x5A),
            "v_scales": Guarded(L.scales_bytes, 0xFF)}
    if not kf:
        bufs["k_scales"] = Guarded(L.scales_bytes, 0xFF)
    ks = None if kf else bufs["k_scales"].as16()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    # prefill through batch-1 views (rows past each length keep their garbage), then one batched append
    l1 = tq.tq_cache_layout_kv(1, max_seq, Hkv, Hkv * G, D, k_format)
    kst, cs, ss = int(L.k_stride_seq), int(L.code_stride_seq), int(L.scale_stride_seq)
    zero = torch.zeros(1, dtype=torch.int32, device="cuda")
    pre = [n - 1 if n == max_seq else n for n in lens]  # leave room for the batched append
    for b in range(B):
        tq.tq_quantize_append(l1, t.k[b][None, :pre[b]].cuda().contiguous(), t.v[b][None, :pre[b]].cuda().contiguous(),
                              pre[b], zero, bufs["k"].view[b * kst:(b + 1) * kst], None if kf else ks[b * ss:],
                              bufs["v_codes"].view[b * cs:(b + 1) * cs], bufs["v_scales"].as16()[b * ss:], status)
    kn = torch.stack([t.k[b][min(pre[b], lens[b] - 1)] for b in range(B)])[:, None]
    vn = torch.stack([t.v[b][min(pre[b], lens[b] - 1)] for b in range(B)])[:, None]
    sp = torch.tensor(pre, dtype=torch.int32, device="cuda")
    tq.tq_quantize_append(L, kn.cuda().contiguous(), vn.cuda().contiguous(), 1, sp, bufs["k"].view, ks,
                          bufs["v_codes"].view, bufs["v_scales"].as16(), status)
    fin = [p + 1 for p in pre]  # every sequence grew by one token (the first one reaches max_seq)
    ws, out = decode_buffers(L, B, Hkv * G, D)
    bufs.update(ws=ws, out=out)
    tq.tq_decode_attention(L, t.q.cuda(), torch.tensor(fin, dtype=torch.int32, device="cuda"), bufs["k"].view, ks,
                           bufs["v_codes"].view, bufs["v_scales"].as16(), w.scale, out.as32f(), ws.view, status)
    all_intact(bufs)
    assert int(status.item()) == 0
    # the oracle on clean caches with the same tokens
    orc = OracleCache(B, max_seq, Hkv, D, kf16=kf)
    parallel_map(lambda b: orc.append_seq(b, t.k[b][:pre[b]], t.v[b][:pre[b]], 0), [b for b in range(B) if pre[b]])
    for b in range(B):
        orc.append_seq(b, kn[b], vn[b], pre[b])
    ref, st = orc.decode_all(t.q, fin, w.scale)
    assert st == 0
    assert_close(out.as32f().view(B, Hkv * G, D).cpu().numpy(), ref, what=f"guards G{G} k{k_format}")


def test_guards_delegated_cache():
    W, F = 64, 16
    lens = [1, 63, 64, 65, 80, 81, 600]
    B, Hkv, G, D = len(lens), 8, 4, 128
    max_seq = 600
    w = syn.Workload("guards_deleg", B, Hkv * G, Hkv, D, lens, torch.bfloat16, 72, max_seq=max_seq)
    t = syn.generate(w)
    L = tq.tq_cache_layout_delegated(B, max_seq, Hkv, Hkv * G, D, W, F)
    bufs = {"k16": Guarded(L.k_bytes, 0x5A), "v_codes": Guarded(L.codes_bytes, 0x5A),
            "v_scales": Guarded(L.scales_bytes, 0xFF), "tail": Guarded(L.tail_bytes, 0xFF)}
    l1 = tq.tq_cache_layout_delegated(1, max_seq, Hkv, Hkv * G, D, W, F)
    kst, cs, ss, ts = int(L.k_stride_seq), int(L.code_stride_seq), int(L.scale_stride_seq), int(L.tail_stride_seq)
    zero = torch.zeros(1, dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for b in range(B):
        tq.tq_append_delegated(l1, t.k[b][None].cuda().contiguous(), t.v[b][None].cuda().contiguous(), lens[b], zero,
                               bufs["k16"].as16()[b * kst // 2:(b + 1) * kst // 2],
                               bufs["v_codes"].view[b * cs:(b + 1) * cs], bufs["v_scales"].as16()[b * ss:],
                               bufs["tail"].as16()[b * ts // 2:(b + 1) * ts // 2], status)
    ws, out = decode_buffers(L, B, Hkv * G, D)
    bufs.update(ws=ws, out=out)
    tq.tq_decode_attention_delegated(L, t.q.cuda(), torch.tensor(lens, dtype=torch.int32, device="cuda"),
                                     bufs["k16"].as16(), bufs["v_codes"].view, bufs["v_scales"].as16(),
                                     bufs["tail"].as16(), w.scale, out.as32f(), ws.view, status)
    all_intact(bufs)
    assert int(status.item()) == 0
    orc = DelegatedOracleCache(B, max_seq, Hkv, D, W, F)
    parallel_map(lambda b: orc.append_seq(b, t.k[b], t.v[b], 0), range(B))
    ref, st = orc.decode_all(t.q, lens, w.scale)
    assert st == 0
    assert_close(out.as32f().view(B, Hkv * G, D).cpu().numpy(), ref, what="guards delegated")


@pytest.mark.parametrize("k_format,unmapped", [(tq.TQ_K_INT4, False), (tq.TQ_K_FP16, False), (tq.TQ_K_INT4, True)])
def test_guards_paged_pools(k_format, unmapped):
    P, max_seq = 64, 640
    lens = [max_seq, 1, 63, 64, 65, 300]
    B, Hkv, G, D = len(lens), 8, 8, 128
    w = syn.Workload("guards_paged", B, Hkv * G, Hkv, D, lens, torch.bfloat16, 73, max_seq=max_seq)
    t = syn.generate(w)
    kf = k_format == tq.TQ_K_FP16
    max_pages = max_seq // P
    n_pages = B * max_pages
    L = tq.tq_cache_layout_paged(B, max_seq, Hkv, Hkv * G, D, k_format, P, n_pages)
    rng = np.random.default_rng(5)
    table = rng.permutation(n_pages).reshape(B, max_pages).astype(np.int32)
    if unmapped:
        table[0, 3] = -1        # sequence 0 loses a page in the middle of its range
        table[5, 2] = n_pages   # and sequence 5 one past the pool
    bufs = {"k": Guarded(L.k_bytes, 0x5A), "v_codes": Guarded(L.codes_bytes, 0x5A),
            "v_scales": Guarded(L.scales_bytes, 0xFF)}
    if not kf:
        bufs["k_scales"] = Guarded(L.scales_bytes, 0xFF)
    ks = None if kf else bufs["k_scales"].as16()
    dt = torch.from_numpy(table).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    L1 = tq.tq_cache_layout_paged(1, max_seq, Hkv, Hkv * G, D, k_format, P, n_pages)
    zero = torch.zeros(1, dtype=torch.int32, device="cuda")
    for b in range(B):
        tq.tq_quantize_append_paged(L1, t.k[b][None].cuda().contiguous(), t.v[b][None].cuda().contiguous(), lens[b],
                                    zero, dt[b:b + 1], bufs["k"].view, ks, bufs["v_codes"].view,
                                    bufs["v_scales"].as16(), status)
    ws, out = decode_buffers(L, B, Hkv * G, D)
    bufs.update(ws=ws, out=out)
    tq.tq_decode_attention_paged(L, t.q.cuda(), torch.tensor(lens, dtype=torch.int32, device="cuda"), dt,
                                 bufs["k"].view, ks, bufs["v_codes"].view, bufs["v_scales"].as16(), w.scale,
                                 out.as32f(), ws.view, status)
    all_intact(bufs)
    got = out.as32f().view(B, Hkv * G, D).cpu().numpy()
    if unmapped:  # reported, skipped, nothing written outside the buffers, output still finite
        assert int(status.item()) & tq.TQ_STATUS_CAPACITY
        assert np.all(np.isfinite(got))
        return
    assert int(status.item()) == 0
    signs = oracle.sign_vector(0, D)
    pools = oracle.new_pool(n_pages, P, Hkv, D, kf)
    parallel_map(lambda b: oracle.quantize_append_paged(signs, np_f32(t.k[b][None]), np_f32(t.v[b][None]),
                                                        np.zeros(1, np.int32), table[b:b + 1], P, max_seq, pools),
                 range(B))
    qn = np_f32(t.q)
    ref, st = oracle_decode_all(lambda which: oracle.decode_attention_paged(
        signs, qn, np.array(lens, np.int32), table, P, max_seq, pools, w.scale, which), B, Hkv * G)
    assert st == 0
    assert_close(got, ref, what=f"guards paged k{k_format}")
