"""GPU parity for paged storage (block table into page pools).

mlxcel guide, §"Known limitations / paged KV scheduler": the paged decode
storage backend. Through the C ABI, against the oracle's paged functions on the
same seeded inputs and the same block table (a random permutation of the
pool's pages): pool rows bit-exact after prefills and appends that cross page
boundaries; decode within max-abs 2e-3 and relative L2 1e-3; an unmapped page
reports TQ_STATUS_CAPACITY instead of touching memory.
"""
import numpy as np
import pytest
import torch

import oracle
from compressed_domain_attention_b200 import synthetic as syn
from compressed_domain_attention_b200 import tq
from tests.parity_utils import assert_close, np_f32, oracle_decode_all, parallel_map

pytestmark = pytest.mark.gpu


class PagedPair:
    def __init__(self, w, k_format, P, extra_pages=7, seed=0):
        self.w, self.P, self.kf16 = w, P, k_format == tq.TQ_K_FP16
        cap = w.capacity
        max_pages = -(-cap // P)
        n_pages = w.batch * max_pages + extra_pages
        self.L = tq.tq_cache_layout_paged(w.batch, cap, w.n_kv_heads, w.n_q_heads, w.head_dim, k_format, P, n_pages)
        rng = np.random.default_rng(seed)
        self.table = rng.permutation(n_pages)[: w.batch * max_pages].reshape(w.batch, max_pages).astype(np.int32)
        self.dtable = torch.from_numpy(self.table).cuda()
        self.kc, self.ks, self.vc, self.vs = tq.alloc_cache(self.L)
        self.signs = oracle.sign_vector(0, w.head_dim)
        self.pools = oracle.new_pool(n_pages, P, w.n_kv_heads, w.head_dim, self.kf16)
        self.cap = cap

    def append(self, k, v, start, status=None):
        """k, v [B][n][Hkv][D] at per-sequence positions start (list)."""
        sp = torch.tensor(start, dtype=torch.int32, device="cuda")
        tq.tq_quantize_append_paged(self.L, k.cuda().contiguous(), v.cuda().contiguous(), k.shape[1], sp,
                                    self.dtable, self.kc, self.ks, self.vc, self.vs, status)
        st = oracle.quantize_append_paged(self.signs, np_f32(k), np_f32(v), np.array(start, np.int32), self.table,
                                          self.P, self.cap, self.pools)
        return st

    def check_pools(self):
        torch.cuda.synchronize()
        L, H, D = self.L, self.w.n_kv_heads, self.w.head_dim
        rows = L.n_pages * L.page_tokens
        pk, pks, pv, pvs = self.pools
        vc = self.vc.cpu().numpy().reshape(rows, H, D // 2)
        vs = self.vs[: rows * H * D // 32].cpu().numpy().view(np.uint16).reshape(rows, H, D // 32)
        assert np.array_equal(vc, pv) and np.array_equal(vs, pvs)
        if self.kf16:
            assert np.array_equal(self.kc.cpu().numpy().view(np.uint16).reshape(rows, H, D), pk)
        else:
            assert np.array_equal(self.kc.cpu().numpy().reshape(rows, H, D // 2), pk)
            ks = self.ks[: rows * H * D // 32].cpu().numpy().view(np.uint16).reshape(rows, H, D // 32)
            assert np.array_equal(ks, pks)

    def decode(self, q, lens, status=None, which=None, **opts):
        w = self.w
        out = torch.full((w.batch, w.n_q_heads, w.head_dim), float("nan"), dtype=torch.float32, device="cuda")
        ws = tq.alloc_workspace(self.L)
        dl = torch.tensor(lens, dtype=torch.int32, device="cuda")
        tq.tq_decode_attention_paged(self.L, q.cuda().contiguous(), dl, self.dtable, self.kc, self.ks, self.vc,
                                     self.vs, w.scale, out, ws, status, **opts)
        ref, st = oracle.decode_attention_paged(self.signs, np_f32(q), np.array(lens, np.int32), self.table, self.P,
                                                self.cap, self.pools, w.scale, which)
        return out.cpu().numpy(), ref, st


def prefill(pair, t, lens):
    """Append every sequence's prefix in 37-token chunks (so appends cross page boundaries), all sequences
    in one call per chunk: rows past a sequence's length get zero vectors, written identically by the GPU
    and the oracle and never read by the decode."""
    w = pair.w
    T = max(lens)
    for start in range(0, T, 37):  # chunks that cross page boundaries
        n = min(37, T - start)
        k = torch.zeros((w.batch, n, w.n_kv_heads, w.head_dim), dtype=w.dtype)
        v = torch.zeros_like(k)
        for b in range(w.batch):
            m = max(0, min(n, lens[b] - start))
            if m:
                k[b, :m] = t.k[b][start:start + m]
                v[b, :m] = t.v[b][start:start + m]
        assert pair.append(k, v, [start] * w.batch) == 0


@pytest.mark.parametrize("D,Hkv,Hq,k_format,P", [(128, 8, 32, tq.TQ_K_INT4, 64), (128, 8, 64, tq.TQ_K_INT4, 32),
                                                 (128, 8, 32, tq.TQ_K_FP16, 16), (128, 4, 32, tq.TQ_K_INT4, 128),
                                                 (64, 2, 8, tq.TQ_K_INT4, 256), (64, 8, 8, tq.TQ_K_FP16, 64),
                                                 (256, 2, 8, tq.TQ_K_INT4, 256)])
def test_paged_append_and_decode(D, Hkv, Hq, k_format, P):
    lens = [1, P - 1, P, P + 1, 3 * P + 7, 500]
    w = syn.Workload(f"paged_d{D}", len(lens), Hq, Hkv, D, lens, torch.bfloat16, 51)
    w.max_seq = max(lens) + 4
    t = syn.generate(w)
    pair = PagedPair(w, k_format, P, seed=D + Hkv)
    prefill(pair, t, lens)
    pair.check_pools()
    out, ref, st = pair.decode(t.q, lens)
    assert st == 0
    # rows past each length hold the chunks' zero padding; the decode reads only [0, len)
    assert_close(out, ref, what=f"paged D{D} Hkv{Hkv} P{P}")
    # one more token per sequence, crossing pages for some
    kn = torch.randn((w.batch, 1, Hkv, D)).to(w.dtype)
    assert pair.append(kn, kn, lens) == 0
    pair.check_pools()
    lens1 = [x + 1 for x in lens]
    out, ref, _ = pair.decode(t.q, lens1)
    assert_close(out, ref, what=f"paged D{D} after append")
    for opts in ({"max_ctas": 5}, {"min_split_tokens": 16}):
        out2, ref2, _ = pair.decode(t.q, lens1, **opts)
        assert_close(out2, ref2, what=f"paged {opts}")


@pytest.mark.parametrize("k_format", [tq.TQ_K_INT4, tq.TQ_K_FP16])
def test_paged_ragged_serving_all_sequences(k_format):
    # all 32 sequences of the serving workload, 64-token pages scattered over the pool
    w = syn.ragged_serving()
    t = syn.generate(w)
    lens = list(w.seq_lens)
    pair = PagedPair(w, k_format, 64, seed=3)
    L1 = tq.tq_cache_layout_paged(1, pair.cap, w.n_kv_heads, w.n_q_heads, w.head_dim, k_format, 64, pair.L.n_pages)
    zero = torch.zeros(1, dtype=torch.int32, device="cuda")
    for b in range(w.batch):  # prefill sequence by sequence: a one-sequence layout over the same pools, table row b
        tq.tq_quantize_append_paged(L1, t.k[b][None].cuda().contiguous(), t.v[b][None].cuda().contiguous(), lens[b],
                                    zero, pair.dtable[b:b + 1], pair.kc, pair.ks, pair.vc, pair.vs)

    def oracle_prefill(b):  # sequences own disjoint pages, so the oracle's appends run side by side
        return oracle.quantize_append_paged(pair.signs, np_f32(t.k[b][None]), np_f32(t.v[b][None]),
                                            np.zeros(1, np.int32), pair.table[b:b + 1], 64, pair.cap, pair.pools)

    assert all(st == 0 for st in parallel_map(oracle_prefill, range(w.batch)))
    pair.check_pools()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.full((w.batch, w.n_q_heads, w.head_dim), float("nan"), dtype=torch.float32, device="cuda")
    tq.tq_decode_attention_paged(pair.L, t.q.cuda().contiguous(), torch.tensor(lens, dtype=torch.int32).cuda(),
                                 pair.dtable, pair.kc, pair.ks, pair.vc, pair.vs, w.scale, out,
                                 tq.alloc_workspace(pair.L), status)
    qn = np_f32(t.q)
    ref, st = oracle_decode_all(lambda which: oracle.decode_attention_paged(
        pair.signs, qn, np.array(lens, np.int32), pair.table, 64, pair.cap, pair.pools, w.scale, which),
        w.batch, w.n_q_heads)
    torch.cuda.synchronize()
    assert st == 0 and int(status.item()) == 0
    assert_close(out.cpu().numpy(), ref, what="paged ragged serving")


def test_paged_unmapped_page_sets_capacity():
    w = syn.Workload("paged_unmapped", 2, 8, 2, 64, [600, 90], torch.bfloat16, 53)
    t = syn.generate(w)
    pair = PagedPair(w, tq.TQ_K_INT4, 256, seed=1)  # this shape's decode tile is 256 tokens
    prefill(pair, t, w.seq_lens)
    pair.check_pools()
    pair.table[0, 1] = -1  # sequence 0 loses its second page
    pair.dtable = torch.from_numpy(pair.table).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, _, st = pair.decode(t.q, w.seq_lens, status)
    assert int(status.item()) & tq.TQ_STATUS_CAPACITY and st & oracle.STATUS_CAPACITY
    assert np.all(np.isfinite(out))
