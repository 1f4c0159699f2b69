"""GPU parity for the per-channel lambda and the sparse-V threshold (both off by default).

* Open-TQ-Metal abstract (the fused quantiser's steps: transform, per-channel
  lambda, per-group abs-max, int4 pack): codes and scales written with lambda
  bit-exact against the oracle; decode with lambda within the usual tolerance.
* mlxcel guide, §"Sparse-V dequant threshold": with threshold 0 the decode is
  the exact one, bit for bit; with a threshold the output stays within the
  oracle's bound (sum of w |V| over the tokens the rule may drop) of exact
  attention; on a two-cluster input whose dropped set is unambiguous (the
  largest score opens every 16-token block), decoded by one CTA, it equals the
  oracle's sparse result.
"""
import numpy as np
import pytest
import torch

import oracle
from compressed_domain_attention_b200 import synthetic as syn
from compressed_domain_attention_b200 import tq
from tests.parity_utils import GpuCache, assert_close, np_f32, parallel_map

pytestmark = pytest.mark.gpu


def lambdas(D, seed):
    g = torch.Generator("cpu").manual_seed(seed)
    lk = torch.exp(torch.rand(D, generator=g) * 2 - 1)
    lv = torch.exp(torch.rand(D, generator=g) * 2 - 1)
    return lk.float(), lv.float()


def oracle_cache(w, t, lk, lv):
    s = oracle.sign_vector(0, w.head_dim)
    kc, ks = oracle.new_cache(w.batch, w.capacity, w.n_kv_heads, w.head_dim)
    vc, vs = oracle.new_cache(w.batch, w.capacity, w.n_kv_heads, w.head_dim)
    for b in range(w.batch):
        st = oracle.quantize_append_lambda(s, np_f32(t.k[b])[None], np_f32(t.v[b])[None], np.zeros(1, np.int32),
                                           None if lk is None else lk.numpy(), None if lv is None else lv.numpy(),
                                           kc[b:b + 1], ks[b:b + 1], vc[b:b + 1], vs[b:b + 1])
        assert st == 0
    return s, kc, ks, vc, vs


def gpu_prefill(w, t, lk, lv, k_format=tq.TQ_K_INT4):
    gpu = GpuCache(w.batch, w.capacity, w.n_kv_heads, w.n_q_heads, w.head_dim, k_format=k_format)
    for b in range(w.batch):
        l1, kc, ks, vc, vs = gpu.seq_view(b)
        sp = torch.zeros(1, dtype=torch.int32, device="cuda")
        tq.tq_quantize_append(l1, t.k[b][None].cuda().contiguous(), t.v[b][None].cuda().contiguous(),
                              w.seq_lens[b], sp, kc, ks, vc, vs, None, None,
                              lambda_k=None if lk is None else lk.cuda(), lambda_v=None if lv is None else lv.cuda())
    torch.cuda.synchronize()
    return gpu


@pytest.mark.parametrize("D,Hkv,Hq", [(128, 8, 32), (128, 8, 64), (64, 2, 8), (32, 1, 4), (256, 1, 4)])
def test_lambda_append_bit_exact_and_decode(D, Hkv, Hq):
    lens = [1, 31, 32, 33, 500]
    w = syn.Workload(f"lam_d{D}", len(lens), Hq, Hkv, D, lens, torch.bfloat16, 31)
    t = syn.generate(w)
    lk, lv = lambdas(D, 7)
    gpu = gpu_prefill(w, t, lk, lv)
    s, kc, ks, vc, vs = oracle_cache(w, t, lk, lv)
    gk, gks, gv, gvs = gpu.host_arrays()
    for b, n in enumerate(lens):
        assert np.array_equal(gk[b, :n], kc[b, :n]) and np.array_equal(gks[b, :n], ks[b, :n])
        assert np.array_equal(gv[b, :n], vc[b, :n]) and np.array_equal(gvs[b, :n], vs[b, :n])
    out = gpu.decode(t.q.cuda(), lens, w.scale, lambda_k=lk.cuda(), lambda_v=lv.cuda()).cpu().numpy()
    ref, _, st = oracle.decode_attention_ext(s, np_f32(t.q), np.array(lens, np.int32), kc, ks, vc, vs, w.scale,
                                             lk.numpy(), lv.numpy())
    assert st == 0
    assert_close(out, ref, what=f"lambda decode D{D}")


def test_lambda_v_with_binary16_k():
    D, lens = 128, [100, 1000]
    w = syn.Workload("lam_kf16", 2, 32, 8, D, lens, torch.bfloat16, 32)
    t = syn.generate(w)
    _, lv = lambdas(D, 8)
    gpu = gpu_prefill(w, t, None, lv, tq.TQ_K_FP16)
    s, _, _, vc, vs = oracle_cache(w, t, None, lv)  # V codes with lambda; K is binary16
    k16 = np.zeros((2, w.capacity, 8, D), np.uint16)
    for b in range(2):
        k16[b, :lens[b]] = np_f32(t.k[b]).astype(np.float16).view(np.uint16)
    gk, _, gv, gvs = gpu.host_arrays()
    assert np.array_equal(gk, k16) and np.array_equal(gv, vc) and np.array_equal(gvs[:, :, :, :], vs)
    out = gpu.decode(t.q.cuda(), lens, w.scale, lambda_v=lv.cuda()).cpu().numpy()
    ref, _, _ = oracle.decode_attention_ext(s, np_f32(t.q), np.array(lens, np.int32), None, None, vc, vs, w.scale,
                                            None, lv.numpy(), k_f16=k16)
    assert_close(out, ref, what="lambda_v with binary16 K")
    # lambda_k has no meaning for binary16 K
    with pytest.raises(tq.TqError) as exc:
        gpu.decode(t.q.cuda(), lens, w.scale, lambda_k=lv.cuda())
    assert exc.value.code == tq.TQ_ERR_INVALID_ARG


@pytest.mark.parametrize("name,k_format", [("ragged_serving", tq.TQ_K_INT4), ("ragged_serving", tq.TQ_K_FP16),
                                           ("llama31_70b_long", tq.TQ_K_INT4)])
def test_sparse_v_within_the_bound(name, k_format):
    # every q head of every sequence: the output stays within the oracle's bound of exact attention
    w = {"ragged_serving": syn.ragged_serving, "llama31_70b_long": syn.llama31_70b_long}[name]()
    t = syn.generate(w)
    gpu = GpuCache(w.batch, w.capacity, w.n_kv_heads, w.n_q_heads, w.head_dim, k_format=k_format)
    for b in range(w.batch):
        gpu.append_seq(b, t.k[b].cuda(), t.v[b].cuda(), 0)
    lens = list(w.seq_lens)
    q = (t.q.float() * 3.0).to(t.q.dtype)  # sharper weights than the workload's own
    exact = gpu.decode(q.cuda(), lens, w.scale).cpu().numpy()
    same = gpu.decode(q.cuda(), lens, w.scale, sparse_v_threshold=0.0).cpu().numpy()
    assert np.array_equal(exact, same)
    kc, ks, vc, vs = gpu.host_arrays()
    s = oracle.sign_vector(0, w.head_dim)
    kf = k_format == tq.TQ_K_FP16
    qn, ln = np_f32(q), np.array(lens, np.int32)
    hp = w.group if w.batch == 1 else w.n_q_heads  # one long sequence: one task per kv head's query group
    tasks = [(b, h0) for b in range(w.batch) for h0 in range(0, w.n_q_heads, hp)]
    for tau in (1e-6, 1e-3):
        got = gpu.decode(q.cuda(), lens, w.scale, sparse_v_threshold=tau).cpu().numpy()

        def one(task, tau=tau):
            b, h0 = task
            which = np.zeros((w.batch, w.n_q_heads), np.uint8)
            which[b, h0:h0 + hp] = 1
            _, bound, st = oracle.decode_attention_ext(s, qn, ln, None if kf else kc, ks, vc, vs, w.scale, tau=tau,
                                                       which=which, k_f16=kc if kf else None)
            ex, _, st2 = oracle.decode_attention_ext(s, qn, ln, None if kf else kc, ks, vc, vs, w.scale,
                                                     which=which, k_f16=kc if kf else None)
            assert st == 0 and st2 == 0
            return b, h0, ex[b, h0:h0 + hp].copy(), bound[b, h0:h0 + hp].copy()

        for b, h0, e, bd in parallel_map(one, tasks):
            g = got[b, h0:h0 + hp]
            assert np.all(np.isfinite(g))
            assert np.all(np.abs(g - e) <= bd + 2e-3), f"tau {tau}: outside the bound (sequence {b}, heads {h0}+)"


def two_cluster_inputs(G, Hkv, D, T, seed):
    """q rows equal within a group; K along each group's q direction: the first token of
    every 16-token block scores 10 (the maximum), 1/8 of the tokens score 10 - ln 10 (kept at
    threshold 0.01), the rest 10 - ln 1000 (dropped); noise orthogonal to q.
    sm_scale = 1/sqrt(D), |q|^2 = D. A split-K warp starts on a 16- or 32-token unit, so its
    running maximum is the global one from its first unit on, and the dropped set is the
    oracle's."""
    g = torch.Generator("cpu").manual_seed(seed)
    qk = torch.randn((Hkv, D), generator=g).sign()  # +-1 entries: |q|^2 = D
    q = qk.repeat_interleave(G, 0)[None]  # [1][Hq][D]
    u = qk / qk.norm(dim=1, keepdim=True)
    coef = torch.full((T,), 10.0 - np.log(1000.0))
    coef[torch.randperm(T, generator=g)[: T // 8]] = 10.0 - np.log(10.0)
    coef[::16] = 10.0
    noise = torch.randn((T, Hkv, D), generator=g)
    noise = noise - (noise * u[None]).sum(-1, keepdim=True) * u[None]
    # score = (q . k) / sqrt(D) = coef * (q . u) / sqrt(D) = coef, since q . u = |q| = sqrt(D)
    k = coef[:, None, None] * u[None] + noise
    v = torch.randn((T, Hkv, D), generator=g)
    v[coef < 5.0] += 4.0  # the dropped cluster's V has mean 4, so dropping it shows in the output
    return q.float(), k.float(), v.float()


@pytest.mark.parametrize("G,k_format", [(1, tq.TQ_K_INT4), (8, tq.TQ_K_INT4), (4, tq.TQ_K_FP16)])
def test_sparse_v_drops_exactly_the_clear_cases(G, k_format):
    Hkv, D, T = 8, 128, 2048
    qq, k, v = two_cluster_inputs(G, Hkv, D, T, 40 + G)
    gpu = GpuCache(1, T, Hkv, Hkv * G, D, k_format=k_format)
    gpu.append_seq(0, k.cuda(), v.cuda(), 0)
    torch.cuda.synchronize()
    scale = 1.0 / np.sqrt(D)
    tau = 0.01
    got = gpu.decode(qq.cuda(), [T], scale, sparse_v_threshold=tau, max_ctas=1).cpu().numpy()
    exact = gpu.decode(qq.cuda(), [T], scale).cpu().numpy()
    kc, ks, vc, vs = gpu.host_arrays()
    s = oracle.sign_vector(0, D)
    kf = k_format == tq.TQ_K_FP16
    ref, bound, _ = oracle.decode_attention_ext(s, qq.numpy(), np.array([T], np.int32), None if kf else kc, ks, vc,
                                                vs, scale, tau=tau, k_f16=kc if kf else None)
    assert_close(got, ref, what=f"sparse-V two clusters G{G}")
    assert np.abs(exact - got).max() > 10 * 2e-3  # the rule dropped a visible share of the weight


def test_sparse_v_argument_errors():
    gpu = GpuCache(1, 64, 1, 4, 64)
    q = torch.zeros((1, 4, 64), dtype=torch.bfloat16, device="cuda")
    for bad in (-1.0, float("nan"), float("inf")):
        with pytest.raises(tq.TqError) as exc:
            gpu.decode(q, [8], 0.1, sparse_v_threshold=bad)
        assert exc.value.code == tq.TQ_ERR_INVALID_ARG
