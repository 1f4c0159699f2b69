"""GPU parity for the delegated hot/cold cache (binary16 K, binary16 V tail folded into int4 V).

mlxcel "TurboQuant KV cache compression", §"Cache modes" (turbo4-delegated: K in
FP16, V as an FP16 hot tail plus a 4-bit cold body) and §"Delegated cache
variant". Through the C ABI, against the oracle's delegated functions on the
same seeded inputs:

* K binary16 bits, the int4 body below the cold length and the tail slots of
  the hot tokens bit-exact, after prefills, single-token steps across fold
  boundaries and multi-token appends longer than the window;
* decode within max-abs 2e-3 and relative L2 1e-3 of the oracle's output.
"""
import numpy as np
import pytest
import torch

from compressed_domain_attention_b200 import synthetic as syn
from compressed_domain_attention_b200 import tq
from tests.parity_utils import (DelegatedGpuCache, DelegatedOracleCache, assert_close,
                                assert_delegated_caches_equal, parallel_map)

pytestmark = pytest.mark.gpu


def build(w, W, F, extra=0):
    t = syn.generate(w)
    cap = w.capacity + extra
    gpu = DelegatedGpuCache(w.batch, cap, w.n_kv_heads, w.n_q_heads, w.head_dim, W, F)
    orc = DelegatedOracleCache(w.batch, cap, w.n_kv_heads, w.head_dim, W, F)
    seqs = list(range(w.batch))
    for b in range(w.batch):
        if w.seq_lens[b]:
            gpu.append_seq(b, t.k[b].cuda(), t.v[b].cuda(), 0)
    parallel_map(lambda b: orc.append_seq(b, t.k[b], t.v[b], 0), [b for b in seqs if w.seq_lens[b]])
    torch.cuda.synchronize()
    return t, gpu, orc, seqs


def check_decode(w, q, gpu, orc, lens, what, **opts):
    """Every sequence and every q head against the oracle."""
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = gpu.decode(q.cuda(), lens, w.scale, status, **opts)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref, st = orc.decode_all(q, lens, w.scale, w.group if w.batch == 1 else None)
    assert st == 0
    return assert_close(out.cpu().numpy(), ref, what=what)


@pytest.mark.parametrize("D,Hkv,Hq,W,F", [(128, 8, 32, 16, 4), (128, 8, 64, 16, 16), (128, 1, 4, 64, 16),
                                          (64, 2, 8, 8, 8), (64, 4, 8, 32, 1), (32, 1, 1, 4, 2),
                                          (32, 8, 64, 16, 8), (128, 2, 16, 1024, 256)])
def test_delegated_prefill_and_decode_shapes(D, Hkv, Hq, W, F):
    # lengths below, at and just past the window, on and off fold boundaries
    lens = [1, W - 1 if W > 1 else 1, W, W + 1, W + F, W + F + 1, 3 * W + 5, 1000]
    w = syn.Workload(f"deleg_d{D}_kv{Hkv}_q{Hq}_w{W}_f{F}", len(lens), Hq, Hkv, D, lens, torch.bfloat16, 21)
    t, gpu, orc, seqs = build(w, W, F)
    assert_delegated_caches_equal(gpu, orc, seqs, w.seq_lens)
    check_decode(w, t.q, gpu, orc, w.seq_lens, f"delegated D{D} Hkv{Hkv} Hq{Hq} W{W} F{F}")


def test_delegated_single_token_steps_cross_fold_boundaries():
    W, F = 16, 4
    lens = [0, 3, 15, 16, 17, 20, 33, 200]
    w = syn.Workload("deleg_steps", len(lens), 32, 8, 128, lens, torch.float16, 22)
    steps = 2 * W + 3
    t, gpu, orc, seqs = build(w, W, F, extra=steps)
    g = torch.Generator("cpu").manual_seed(5)
    cur = list(lens)
    for i in range(steps):
        k = torch.randn((w.batch, 1, 8, 128), generator=g).to(torch.float16)
        v = torch.randn((w.batch, 1, 8, 128), generator=g).to(torch.float16)
        gpu.append_all(k.cuda(), v.cuda(), cur)
        for b in range(w.batch):
            orc.append_seq(b, k[b], v[b], cur[b])
        cur = [x + 1 for x in cur]
        if i % 5 == 4 or i == steps - 1:
            torch.cuda.synchronize()
            assert_delegated_caches_equal(gpu, orc, seqs, cur)
            q = torch.randn((w.batch, 32, 128), generator=g).to(torch.float16)
            check_decode(w, q, gpu, orc, cur, f"delegated step {i}")


@pytest.mark.parametrize("chunks", [[3, 17, 1, 40, 2], [64, 1, 1, 33]])
def test_delegated_multi_token_appends(chunks):
    # appends longer than the window fold old hot tokens whose slots new hot tokens take
    W, F = 16, 8
    lens = [0, 5, 16, 23, 64]
    w = syn.Workload("deleg_chunks", len(lens), 8, 2, 64, lens, torch.float32, 23)
    t, gpu, orc, seqs = build(w, W, F, extra=sum(chunks))
    g = torch.Generator("cpu").manual_seed(6)
    cur = list(lens)
    for n in chunks:
        k = torch.randn((w.batch, n, 2, 64), generator=g)
        v = torch.randn((w.batch, n, 2, 64), generator=g)
        gpu.append_all(k.cuda(), v.cuda(), cur)
        for b in range(w.batch):
            orc.append_seq(b, k[b], v[b], cur[b])
        cur = [x + n for x in cur]
        torch.cuda.synchronize()
        assert_delegated_caches_equal(gpu, orc, seqs, cur)
    q = torch.randn((w.batch, 8, 64), generator=g)
    check_decode(w, q, gpu, orc, cur, "delegated chunks")


def test_delegated_ragged_serving_all_sequences():
    w = syn.ragged_serving()
    t, gpu, orc, seqs = build(w, syn.DELEGATED_WINDOW, syn.DELEGATED_FOLD)
    assert_delegated_caches_equal(gpu, orc, seqs, w.seq_lens)
    check_decode(w, t.q, gpu, orc, w.seq_lens, "delegated ragged serving")
    # the bench's step: one appended token per sequence, then the decode
    cur = list(w.seq_lens)
    gpu.append_all(t.k_new.cuda(), t.v_new.cuda(), cur)
    for b in seqs:
        orc.append_seq(b, t.k_new[b], t.v_new[b], cur[b])
    cur = [x + 1 for x in cur]
    torch.cuda.synchronize()
    assert_delegated_caches_equal(gpu, orc, seqs, cur)
    check_decode(w, t.q, gpu, orc, cur, "delegated ragged serving step")


def test_delegated_long_context_all_heads():
    w = syn.llama31_70b_long()
    W, F = syn.DELEGATED_WINDOW, syn.DELEGATED_FOLD
    t = syn.generate(w)
    gpu = DelegatedGpuCache(1, w.capacity, w.n_kv_heads, w.n_q_heads, w.head_dim, W, F)
    gpu.append_seq(0, t.k[0].cuda(), t.v[0].cuda(), 0)
    orc = DelegatedOracleCache(1, w.capacity, w.n_kv_heads, w.head_dim, W, F)
    orc.append_seq(0, t.k[0], t.v[0], 0)
    torch.cuda.synchronize()
    assert_delegated_caches_equal(gpu, orc, [0], w.seq_lens)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = gpu.decode(t.q.cuda(), w.seq_lens, w.scale, status).cpu().numpy()
    assert int(status.item()) == 0
    ref, st = orc.decode_all(t.q, w.seq_lens, w.scale, w.group)
    assert st == 0
    assert_close(out, ref, what="delegated 131072-token context")


def test_delegated_split_options_agree():
    W, F = 32, 8
    lens = [2000, 700, 40, 0]
    w = syn.Workload("deleg_split", len(lens), 32, 8, 128, lens, torch.bfloat16, 24)
    t, gpu, orc, seqs = build(w, W, F)
    ref, _ = orc.decode(t.q, lens, w.scale)
    q = t.q.cuda()
    for opts in ({}, {"max_ctas": 7}, {"min_split_tokens": 16}, {"max_ctas": 300, "min_split_tokens": 16}):
        out = gpu.decode(q, lens, w.scale, **opts).cpu().numpy()
        assert_close(out, ref, what=f"delegated split {opts}")
    assert np.all(out[3] == 0)  # the empty sequence


def test_delegated_nonfinite_v_and_argument_errors():
    W, F = 8, 4
    gpu = DelegatedGpuCache(1, 16, 1, 4, 64, W, F)
    k = torch.randn((3, 1, 64))
    v = torch.randn((3, 1, 64))
    v[2, 0, 9] = 1.0e6  # beyond binary16: stored as inf in the tail
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    gpu.append_seq(0, k.cuda(), v.cuda(), 0, status)
    torch.cuda.synchronize()
    assert int(status.item()) & tq.TQ_STATUS_NONFINITE
    _, _, _, tail = gpu.host_arrays()
    assert tail[0, 2, 0, 9] == 0x7C00
    # head_dim 256: binary16 K tiles are limited to 128
    L = tq.tq_cache_layout_delegated(1, 64, 1, 4, 256, 8, 4)
    k16, _, vc, vs = tq.alloc_cache(L)
    tl = tq.alloc_tail(L)
    q = torch.zeros((1, 4, 256), dtype=torch.bfloat16, device="cuda")
    lens = torch.tensor([8], dtype=torch.int32, device="cuda")
    out = torch.zeros((1, 4, 256), dtype=torch.float32, device="cuda")
    with pytest.raises(tq.TqError) as exc:
        tq.tq_decode_attention_delegated(L, q, lens, k16, vc, vs, tl, 0.1, out, tq.alloc_workspace(L))
    assert exc.value.code == tq.TQ_ERR_UNSUPPORTED
    # a missing tail
    L2 = gpu.layout
    q2 = torch.zeros((1, 4, 64), dtype=torch.bfloat16, device="cuda")
    out2 = torch.zeros((1, 4, 64), dtype=torch.float32, device="cuda")
    with pytest.raises(tq.TqError) as exc:
        tq.tq_decode_attention_delegated(L2, q2, lens, gpu.k16, gpu.v_codes, gpu.v_scales, None, 0.1, out2,
                                         tq.alloc_workspace(L2))
    assert exc.value.code == tq.TQ_ERR_INVALID_ARG
