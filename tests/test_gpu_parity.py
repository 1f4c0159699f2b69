"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

* codes and binary16 scale bits must be bit-exact;
* decode output within max-abs 2e-3 and relative L2 1e-3 of the oracle's fp32
  result on the oracle's own (bit-identical) cache.

Workloads: the seeded synthetic recipes of ``compressed_domain_attention_b200.synthetic``
(tiny single head; Llama-3-8B-shaped layer; Gemma-3-1B sweep; Llama-3.1-70B-shaped
131K context; 32-sequence ragged serving), plus ragged / degenerate edge cases.
"""
import numpy as np
import pytest
import torch

from compressed_domain_attention_b200 import synthetic as syn
from compressed_domain_attention_b200 import tq
from tests.parity_utils import GpuCache, OracleCache, assert_close, np_f32

pytestmark = pytest.mark.gpu


def fill_both(w, t, gpu, orc):
    """Prefill every sequence, on the GPU and in the oracle (a host thread pool)."""
    for b in range(w.batch):
        if w.seq_lens[b] == 0 or t.k[b] is None:
            continue
        gpu.append_seq(b, t.k[b].cuda(), t.v[b].cuda(), 0)
    orc.append_seqs(t, [b for b in range(w.batch) if w.seq_lens[b]])


def compare_caches(gpu, orc, seqs, lens):
    kc, ks, vc, vs = gpu.host_arrays()
    for b in seqs:
        L = lens[b]
        assert np.array_equal(kc[b, :L], orc.kc[b, :L]), f"K codes differ in sequence {b}"
        assert np.array_equal(vc[b, :L], orc.vc[b, :L]), f"V codes differ in sequence {b}"
        assert np.array_equal(ks[b, :L], orc.ks[b, :L]), f"K scales differ in sequence {b}"
        assert np.array_equal(vs[b, :L], orc.vs[b, :L]), f"V scales differ in sequence {b}"


def run_workload(w, check_append=True):
    """Every sequence and every q head of the workload against the oracle."""
    t = syn.generate(w)
    cap = w.capacity
    gpu = GpuCache(w.batch, cap, w.n_kv_heads, w.n_q_heads, w.head_dim)
    orc = OracleCache(w.batch, cap, w.n_kv_heads, w.head_dim)
    fill_both(w, t, gpu, orc)
    torch.cuda.synchronize()
    seqs = list(range(w.batch))
    compare_caches(gpu, orc, seqs, w.seq_lens)
    q = t.q.cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = gpu.decode(q, w.seq_lens, w.scale, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    hpt = w.group if w.batch == 1 else None  # one long sequence: one task per kv head's query group
    ref, st = orc.decode_all(t.q, w.seq_lens, w.scale, hpt)
    assert st == 0
    got = out.cpu().numpy()
    res = assert_close(got, ref, what=w.name)
    print(f"\n{w.name}: max_abs {res[0]:.3e} rel_l2 {res[1]:.3e}")
    if check_append and w.n_append:
        # append one token per sequence at its length, then decode over len + 1
        lens1 = [L + w.n_append for L in w.seq_lens]
        gpu.append_all(t.k_new.cuda(), t.v_new.cuda(), w.seq_lens, status)
        for b in seqs:
            orc.append_seq(b, t.k_new[b], t.v_new[b], w.seq_lens[b])
        torch.cuda.synchronize()
        compare_caches(gpu, orc, seqs, lens1)
        out1 = gpu.decode(q, lens1, w.scale, status)
        ref1, _ = orc.decode_all(t.q, lens1, w.scale, hpt)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert_close(out1.cpu().numpy(), ref1, what=w.name + " +append")
    return res


def test_tiny_single_head():
    run_workload(syn.tiny_single_head())


def test_llama3_8b_layer():
    run_workload(syn.llama3_8b_layer())


@pytest.mark.parametrize("T", syn.GEMMA_SWEEP)
def test_gemma3_1b_sweep(T):
    run_workload(syn.gemma3_1b_sweep(T))


def test_llama31_70b_long_context():
    run_workload(syn.llama31_70b_long())


def test_ragged_serving_all_sequences():
    # all 32 sequences (about 0.55 M tokens) and all 32 q heads of each
    run_workload(syn.ragged_serving())


def test_ragged_serving_prefill_4096():
    # the serving workload's 4096-token prefill quantise of one sequence, bit-exact
    w = syn.Workload("prefill_4096_gqa4_d128_bf16", 1, 32, 8, 128, [4096], torch.bfloat16, 4)
    t = syn.generate(w)
    gpu = GpuCache(1, 4096, 8, 32, 128)
    orc = OracleCache(1, 4096, 8, 128)
    gpu.append_seq(0, t.k[0].cuda(), t.v[0].cuda(), 0)
    orc.append_seq(0, t.k[0], t.v[0], 0)
    torch.cuda.synchronize()
    compare_caches(gpu, orc, [0], [4096])


# ----------------------------------------------------------------------------- shapes and edge cases

def random_case(B, lens, Hkv, G, D, dtype=torch.bfloat16, seed=0, cap=None, sm_scale=None):
    w = syn.Workload(f"case_b{B}_h{Hkv}x{G}_d{D}", B, Hkv * G, Hkv, D, list(lens), dtype, seed,
                     max_seq=cap or max(max(lens), 1), sm_scale=sm_scale)
    t = syn.generate(w)
    gpu = GpuCache(B, w.capacity, Hkv, Hkv * G, D)
    orc = OracleCache(B, w.capacity, Hkv, D)
    fill_both(w, t, gpu, orc)
    return w, t, gpu, orc


@pytest.mark.parametrize("D", [32, 64, 128, 256])
@pytest.mark.parametrize("Hkv,G", [(1, 1), (1, 8), (2, 3), (4, 2), (8, 1), (8, 8)])
def test_shapes(D, Hkv, G):
    lens = [1, 37, 300]
    w, t, gpu, orc = random_case(3, lens, Hkv, G, D, seed=D + 10 * Hkv + G)
    torch.cuda.synchronize()
    compare_caches(gpu, orc, range(3), lens)
    out = gpu.decode(t.q.cuda(), lens, w.scale)
    ref, _ = orc.decode(t.q, lens, w.scale)
    assert_close(out.cpu().numpy(), ref, what=w.name)


def test_ragged_edge_lengths():
    # lengths around the 16-token unit, the stage tile and the split range,
    # including empty and full sequences
    lens = [0, 1, 15, 16, 17, 31, 32, 33, 127, 128, 129, 255, 256, 257, 1000, 2048]
    w, t, gpu, orc = random_case(len(lens), lens, 8, 4, 128, seed=7, cap=2048)
    out = gpu.decode(t.q.cuda(), lens, w.scale)
    ref, _ = orc.decode(t.q, lens, w.scale)
    got = out.cpu().numpy()
    assert np.all(got[0] == 0.0)  # empty sequence -> zero output
    assert_close(got, ref, what="ragged edges")


@pytest.mark.parametrize("max_ctas,min_split", [(1, 16), (3, 16), (7, 64), (148, 128), (300, 16), (1024, 16),
                                               (148, 100000)])
def test_split_invariance(max_ctas, min_split):
    lens = [4096]
    w, t, gpu, orc = random_case(1, lens, 8, 4, 128, seed=1)
    out = gpu.decode(t.q.cuda(), lens, w.scale, max_ctas=max_ctas, min_split_tokens=min_split)
    ref, _ = orc.decode(t.q, lens, w.scale)
    assert_close(out.cpu().numpy(), ref, what=f"grid {max_ctas} min_split {min_split}")


def test_multi_sequence_per_cta():
    # many short sequences: CTA ranges straddle sequence boundaries
    lens = [int(x) for x in np.random.default_rng(3).integers(0, 90, size=64)]
    w, t, gpu, orc = random_case(64, lens, 2, 4, 64, seed=11, cap=96)
    out = gpu.decode(t.q.cuda(), lens, w.scale, max_ctas=5, min_split_tokens=16)
    ref, _ = orc.decode(t.q, lens, w.scale)
    assert_close(out.cpu().numpy(), ref, what="straddling ranges")


def test_maximum_batch():
    # the largest batch the decode takes, 1024 sequences: block-wide prefix sums with
    # several lengths per thread, default-grid ranges straddling many sequences, empty
    # sequences among them; then one batched append of a token to every sequence
    # (start = its length) and the decode over len + 1
    rng = np.random.default_rng(21)
    lens = [int(x) for x in rng.integers(0, 41, size=1024)]
    lens[0] = lens[511] = 0
    lens[1023] = 47
    Hkv, G, D = 2, 2, 64
    w, t, gpu, orc = random_case(1024, lens, Hkv, G, D, seed=21, cap=48)
    out = gpu.decode(t.q.cuda(), lens, w.scale)
    ref, _ = orc.decode(t.q, lens, w.scale)
    got = out.cpu().numpy()
    assert np.all(got[[0, 511]] == 0.0)
    assert_close(got, ref, what="batch 1024")

    g = torch.Generator().manual_seed(22)
    k1 = torch.randn((1024, 1, Hkv, D), generator=g).to(torch.bfloat16)
    v1 = torch.randn((1024, 1, Hkv, D), generator=g).to(torch.bfloat16)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    gpu.append_all(k1.cuda(), v1.cuda(), lens, status)
    for b in range(1024):
        orc.append_seq(b, k1[b], v1[b], lens[b])
    lens1 = [L + 1 for L in lens]
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    compare_caches(gpu, orc, range(1024), lens1)
    out1 = gpu.decode(t.q.cuda(), lens1, w.scale)
    ref1, _ = orc.decode(t.q, lens1, w.scale)
    assert_close(out1.cpu().numpy(), ref1, what="batch 1024 + append")


@pytest.mark.parametrize("qdt", [torch.float32, torch.float16, torch.bfloat16])
def test_query_dtypes(qdt):
    lens = [500, 1]
    w, t, gpu, orc = random_case(2, lens, 4, 4, 128, seed=5)
    q = t.q.to(qdt)
    out = gpu.decode(q.cuda(), lens, w.scale)
    ref, _ = orc.decode(q, lens, w.scale)
    assert_close(out.cpu().numpy(), ref, what=str(qdt))


def test_attention_scale_one():
    # Gemma-4-style attn_scale = 1.0 (Open-TQ-Metal arXiv abstract)
    lens = [700]
    w, t, gpu, orc = random_case(1, lens, 2, 4, 128, seed=9, sm_scale=1.0)
    out = gpu.decode(t.q.cuda(), lens, 1.0)
    ref, _ = orc.decode(t.q, lens, 1.0)
    assert_close(out.cpu().numpy(), ref, what="sm_scale 1.0")


def test_fp32_inputs_bitexact_and_nonfinite():
    D, Hkv = 128, 2
    gpu = GpuCache(2, 8, Hkv, Hkv, D)
    orc = OracleCache(2, 8, Hkv, D)
    g = torch.Generator().manual_seed(0)
    k = torch.randn((3, Hkv, D), generator=g) * 100
    v = torch.randn((3, Hkv, D), generator=g)
    k[1, 0, 5] = float("inf")
    v[2, 1, 7] = 1e30
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    gpu.append_seq(1, k.cuda(), v.cuda(), 2, status)
    torch.cuda.synchronize()
    assert int(status.item()) & tq.TQ_STATUS_NONFINITE
    import oracle
    st = oracle.quantize_append(orc.signs, np_f32(k)[None], np_f32(v)[None], np.array([2], np.int32),
                                orc.kc[1:2], orc.ks[1:2], orc.vc[1:2], orc.vs[1:2])
    assert st & oracle.STATUS_NONFINITE
    compare_caches(gpu, orc, [0, 1], [8, 8])


def test_append_capacity_status_and_skip():
    D, Hkv = 64, 1
    gpu = GpuCache(2, 10, Hkv, Hkv, D)
    g = torch.Generator().manual_seed(1)
    k = torch.randn((2, 4, Hkv, D), generator=g).to(torch.bfloat16).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    gpu.append_all(k, k, [6, 7], status)  # 7 + 4 > 10: sequence 1 skipped
    torch.cuda.synchronize()
    assert int(status.item()) & tq.TQ_STATUS_CAPACITY
    kc, ks, _, _ = gpu.host_arrays()
    assert np.any(kc[0, 6:10] != 0) and np.all(kc[1] == 0) and np.all(ks[1] == 0)


def test_decode_length_out_of_range_status():
    lens = [40, 40]
    w, t, gpu, orc = random_case(2, lens, 1, 1, 128, seed=2)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = gpu.decode(t.q.cuda(), [41, 40], w.scale, status)  # 41 > max_seq: treated as empty
    torch.cuda.synchronize()
    assert int(status.item()) & tq.TQ_STATUS_CAPACITY
    got = out.cpu().numpy()
    assert np.all(got[0] == 0)
    ref, _ = orc.decode(t.q, [0, 40], w.scale)
    assert_close(got, ref, what="length out of range")


@pytest.mark.parametrize("domain", [0, 1])
def test_dequantize_debug_bitexact(domain):
    import oracle
    lens = [50, 3]
    w, t, gpu, orc = random_case(2, lens, 2, 1, 128, seed=4, cap=64)
    out = torch.empty((2, 64, 2, 128), dtype=torch.float32, device="cuda")
    tq.tq_dequantize_debug(gpu.layout, gpu.k_codes, gpu.k_scales, torch.tensor(lens, dtype=torch.int32).cuda(),
                           domain, out)
    ref, _ = oracle.dequantize(orc.signs, orc.kc, orc.ks, np.array(lens, np.int32), bool(domain))
    assert np.array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32))


def test_no_dequantised_buffer_in_workspace():
    # Open-TQ-Metal: no intermediate dequantised K/V. The workspace holds only
    # O(splits * heads * D) partials, independent of the context length.
    small = tq.tq_cache_layout(1, 1024, 8, 64, 128)
    large = tq.tq_cache_layout(1, 131072, 8, 64, 128)
    assert small.decode_workspace_bytes == large.decode_workspace_bytes
    assert large.decode_workspace_bytes < 131072 * 8 * 128 * 2  # far below one dense bf16 K


def test_repeated_calls_deterministic():
    lens = [3000, 17]
    w, t, gpu, orc = random_case(2, lens, 8, 8, 128, seed=8)
    a = gpu.decode(t.q.cuda(), lens, w.scale).cpu()
    b = gpu.decode(t.q.cuda(), lens, w.scale).cpu()
    assert torch.equal(a, b)
