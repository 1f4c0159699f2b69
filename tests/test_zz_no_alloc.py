"""tq_decode_attention_noalloc: decode for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc when they decode (inside a memory pool or
custom allocator that must not re-enter itself, under a fixed device-memory
plan, or as a plug-in handed only its tensors). This entry point takes its
split-K scratch from a fixed array in the library's device image instead of a
caller workspace. Through the C ABI, two calls in a row must match the regular
entry point (which uses a caller workspace) within the decode tolerance, and
the oracle too; a binary16-K (asymmetric) cache goes through the same shared
scratch; a request larger than the array must be refused.

This file is collected last on purpose, and it also passes alone in a fresh
process (the first call on the device sets up the array's address).
"""
import numpy as np
import pytest
import torch

from compressed_domain_attention_b200 import synthetic as syn
from compressed_domain_attention_b200 import tq
from tests.parity_utils import ATOL, RTOL_L2, GpuCache, OracleCache, assert_close

pytestmark = pytest.mark.gpu


def build_case(k_format=tq.TQ_K_INT4, seed=21):
    lens = [3000, 1, 257, 1400]
    w = syn.Workload(f"noalloc_b4_gqa4_d128_k{k_format}", 4, 32, 8, 128, lens, torch.bfloat16, seed)
    t = syn.generate(w)
    gpu = GpuCache(w.batch, w.capacity, w.n_kv_heads, w.n_q_heads, w.head_dim, k_format=k_format)
    orc = OracleCache(w.batch, w.capacity, w.n_kv_heads, w.head_dim, kf16=k_format == tq.TQ_K_FP16)
    for b in range(w.batch):
        gpu.append_seq(b, t.k[b].cuda(), t.v[b].cuda(), 0)
    orc.append_seqs(t, range(w.batch))
    return w, t, gpu, orc


@pytest.mark.parametrize("k_format", [tq.TQ_K_INT4, tq.TQ_K_FP16])
def test_noalloc_matches_workspace_entry_point_and_oracle_twice(k_format):
    w, t, gpu, orc = build_case(k_format)
    q = t.q.cuda()
    lens = torch.tensor(w.seq_lens, dtype=torch.int32, device="cuda")
    ref_ws = gpu.decode(q, w.seq_lens, w.scale).cpu().numpy()  # regular entry point, caller workspace
    ref, st = orc.decode_all(t.q, w.seq_lens, w.scale)
    assert st == 0
    for _ in range(2):  # the scratch keeps the previous call's contents; results must not depend on them
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        out = torch.full((w.batch, w.n_q_heads, w.head_dim), float("nan"), dtype=torch.float32, device="cuda")
        tq.tq_decode_attention_noalloc(gpu.layout, q, lens, gpu.k_codes, gpu.k_scales, gpu.v_codes, gpu.v_scales,
                                       w.scale, out, status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        got = out.cpu().numpy()
        assert_close(got, ref_ws, ATOL, RTOL_L2, what="no-alloc vs workspace entry point")
        assert_close(got, ref, ATOL, RTOL_L2, what="no-alloc vs oracle")


def test_noalloc_refuses_requests_beyond_the_scratch():
    # (SMs + 1024) slots x 64 q heads x (128 + 2) floats is far above the scratch size
    L = tq.tq_cache_layout(1024, 16, 8, 64, 128)
    d = torch.zeros(16, dtype=torch.uint8, device="cuda")
    f = torch.zeros(16, dtype=torch.float32, device="cuda")
    i = torch.zeros(1024, dtype=torch.int32, device="cuda")
    with pytest.raises(tq.TqError) as exc:
        tq.tq_decode_attention_noalloc(L, f, i, d, d, d, d, 0.1, f)
    assert exc.value.code == tq.TQ_ERR_CAPACITY
    assert np.isfinite(ATOL)
