"""GPU parity for the asymmetric cache (binary16 K in the original domain, int4 V).

mlxcel "TurboQuant KV cache compression", §"Cache modes": the recommended
default keeps K in FP16 and compresses only V. Through the C ABI, against the
oracle's asymmetric functions on the same seeded inputs:

* K binary16 bits, V codes and V scale bits bit-exact;
* decode within max-abs 2e-3 and relative L2 1e-3 of the oracle's fp32 output.

Shapes cover both score layouts (query groups of <= 4 heads and of 8), every
head_dim the format supports, ragged lengths with tile and unit edges, and the
131072-token long-context shape (every head of every sequence).
"""
import numpy as np
import pytest
import torch

from compressed_domain_attention_b200 import synthetic as syn
from compressed_domain_attention_b200 import tq
from tests.parity_utils import GpuCache, OracleCache, assert_close

pytestmark = pytest.mark.gpu


def build(w):
    t = syn.generate(w)
    cap = w.capacity
    gpu = GpuCache(w.batch, cap, w.n_kv_heads, w.n_q_heads, w.head_dim, k_format=tq.TQ_K_FP16)
    orc = OracleCache(w.batch, cap, w.n_kv_heads, w.head_dim, kf16=True)
    seqs = list(range(w.batch))
    for b in range(w.batch):
        if w.seq_lens[b]:
            gpu.append_seq(b, t.k[b].cuda(), t.v[b].cuda(), 0)
    orc.append_seqs(t, [b for b in seqs if w.seq_lens[b]])
    torch.cuda.synchronize()
    return t, gpu, orc, seqs


def check_caches(gpu, orc, seqs, lens):
    kc, _, vc, vs = gpu.host_arrays()
    for b in seqs:
        n = lens[b]
        assert np.array_equal(kc[b, :n], orc.kc[b, :n]), f"binary16 K differs in sequence {b}"
        assert np.array_equal(vc[b, :n], orc.vc[b, :n]), f"V codes differ in sequence {b}"
        assert np.array_equal(vs[b, :n], orc.vs[b, :n]), f"V scales differ in sequence {b}"


def check_decode(w, t, gpu, orc, what):
    """Every sequence and every q head against the oracle."""
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = gpu.decode(t.q.cuda(), w.seq_lens, w.scale, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref, st = orc.decode_all(t.q, w.seq_lens, w.scale, w.group if w.batch == 1 else None)
    assert st == 0
    return assert_close(out.cpu().numpy(), ref, what=what)


@pytest.mark.parametrize("D,Hkv,Hq", [(128, 8, 32), (128, 8, 64), (128, 1, 4), (128, 2, 16), (64, 2, 8),
                                      (64, 4, 8), (32, 1, 1), (32, 8, 64)])
def test_kf16_append_and_decode_shapes(D, Hkv, Hq):
    lens = [1, 15, 16, 17, 33, 300, 1000]
    w = syn.Workload(f"kf16_d{D}_kv{Hkv}_q{Hq}", len(lens), Hq, Hkv, D, lens, torch.bfloat16, 11)
    t, gpu, orc, seqs = build(w)
    check_caches(gpu, orc, seqs, w.seq_lens)
    check_decode(w, t, gpu, orc, f"kf16 D{D} Hkv{Hkv} Hq{Hq}")


@pytest.mark.parametrize("name", ["llama3_8b_layer", "ragged_serving"])
def test_kf16_workload_shapes(name):
    w = {"llama3_8b_layer": syn.llama3_8b_layer, "ragged_serving": syn.ragged_serving}[name]()
    t, gpu, orc, seqs = build(w)
    check_caches(gpu, orc, seqs, w.seq_lens)
    check_decode(w, t, gpu, orc, f"kf16 {w.name}")


def test_kf16_long_context_all_heads():
    w = syn.llama31_70b_long()
    t = syn.generate(w)
    gpu = GpuCache(1, w.capacity, w.n_kv_heads, w.n_q_heads, w.head_dim, k_format=tq.TQ_K_FP16)
    gpu.append_seq(0, t.k[0].cuda(), t.v[0].cuda(), 0)
    orc = OracleCache(1, w.capacity, w.n_kv_heads, w.head_dim, kf16=True)
    orc.append_seq(0, t.k[0], t.v[0], 0)
    torch.cuda.synchronize()
    kc, _, vc, vs = gpu.host_arrays()
    assert np.array_equal(kc, orc.kc) and np.array_equal(vc, orc.vc) and np.array_equal(vs, orc.vs)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = gpu.decode(t.q.cuda(), w.seq_lens, w.scale, status).cpu().numpy()
    assert int(status.item()) == 0
    ref, st = orc.decode_all(t.q, w.seq_lens, w.scale, w.group)
    assert st == 0
    assert_close(out, ref, what="kf16 131072-token context")


def test_kf16_split_invariance_and_append_then_decode():
    lens = [2000, 700]
    w = syn.Workload("kf16_split", 2, 32, 8, 128, lens, torch.bfloat16, 12, n_append=3)
    t, gpu, orc, seqs = build(w)
    # append 3 more tokens per sequence through the batched call, then decode over them
    sp = [lens[0], lens[1]]
    gpu.append_all(t.k_new.cuda(), t.v_new.cuda(), sp)
    for b in range(2):
        orc.append_seq(b, t.k_new[b], t.v_new[b], sp[b])
    torch.cuda.synchronize()
    new_lens = [x + 3 for x in lens]
    check_caches(gpu, orc, [0, 1], new_lens)
    ref, _ = orc.decode(t.q, new_lens, w.scale)
    q = t.q.cuda()
    outs = []
    for opts in ({}, {"max_ctas": 7}, {"min_split_tokens": 16}, {"max_ctas": 300, "min_split_tokens": 16}):
        out = gpu.decode(q, new_lens, w.scale, **opts).cpu().numpy()
        assert_close(out, ref, what=f"kf16 split {opts}")
        outs.append(out)


def test_kf16_rejects_head_dim_256_and_missing_buffers():
    L = tq.tq_cache_layout_kv(1, 64, 1, 4, 256, tq.TQ_K_FP16)
    kc, ks, vc, vs = tq.alloc_cache(L)
    assert ks is None
    q = torch.zeros((1, 4, 256), dtype=torch.bfloat16, device="cuda")
    lens = torch.tensor([8], dtype=torch.int32, device="cuda")
    out = torch.zeros((1, 4, 256), dtype=torch.float32, device="cuda")
    with pytest.raises(tq.TqError) as exc:
        tq.tq_decode_attention(L, q, lens, kc, ks, vc, vs, 0.1, out, tq.alloc_workspace(L))
    assert exc.value.code == tq.TQ_ERR_UNSUPPORTED
    # the symmetric format still needs its K scales
    L4 = tq.tq_cache_layout(1, 64, 1, 4, 128)
    kc4, _, vc4, vs4 = tq.alloc_cache(L4)
    q4 = torch.zeros((1, 4, 128), dtype=torch.bfloat16, device="cuda")
    out4 = torch.zeros((1, 4, 128), dtype=torch.float32, device="cuda")
    with pytest.raises(tq.TqError) as exc:
        tq.tq_decode_attention(L4, q4, lens, kc4, None, vc4, vs4, 0.1, out4, tq.alloc_workspace(L4))
    assert exc.value.code == tq.TQ_ERR_INVALID_ARG


def test_kf16_nonfinite_k_sets_status():
    w = syn.Workload("kf16_nonfinite", 1, 4, 1, 64, [16], torch.float32, 13)
    t = syn.generate(w)
    k = t.k[0].clone()
    k[3, 0, 5] = 1.0e6  # beyond the binary16 range
    gpu = GpuCache(1, 16, 1, 4, 64, k_format=tq.TQ_K_FP16)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    gpu.append_seq(0, k.cuda(), t.v[0].cuda(), 0, status)
    torch.cuda.synchronize()
    assert int(status.item()) & tq.TQ_STATUS_NONFINITE
    kc, _, _, _ = gpu.host_arrays()
    assert kc[0, 3, 0, 5] == 0x7C00
