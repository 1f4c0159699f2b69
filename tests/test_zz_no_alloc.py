"""tq_decode_attention_noalloc: decode for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc when they decode (inside a memory pool or
custom allocator that must not re-enter itself, under a fixed device-memory
plan, or as a plug-in handed only its tensors). This entry point takes its
split-K scratch from a fixed array in the library's device image instead of a
caller workspace. Through the C ABI, two calls in a row must match the regular
entry point (which uses a caller workspace) within the decode tolerance, and a
request larger than the array must be refused.

This file is collected last on purpose, and it also passes alone in a fresh
process (the first call on the device sets up the array's address).
"""
import numpy as np
import pytest
import torch

from compressed_domain_attention_b200 import synthetic as syn
from compressed_domain_attention_b200 import tq
from tests.parity_utils import ATOL, RTOL_L2, GpuCache, assert_close

pytestmark = pytest.mark.gpu


def build_case():
    lens = [3000, 1, 257, 1400]
    w = syn.Workload("noalloc_b4_gqa4_d128", 4, 32, 8, 128, lens, torch.bfloat16, 21)
    t = syn.generate(w)
    gpu = GpuCache(w.batch, w.capacity, w.n_kv_heads, w.n_q_heads, w.head_dim)
    for b in range(w.batch):
        gpu.append_seq(b, t.k[b].cuda(), t.v[b].cuda(), 0)
    return w, t, gpu


def test_noalloc_matches_workspace_entry_point_twice():
    w, t, gpu = build_case()
    q = t.q.cuda()
    lens = torch.tensor(w.seq_lens, dtype=torch.int32, device="cuda")
    ref = gpu.decode(q, w.seq_lens, w.scale).cpu().numpy()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for _ in range(2):  # the scratch keeps the previous call's contents; results must not depend on them
        out = torch.full((w.batch, w.n_q_heads, w.head_dim), float("nan"), dtype=torch.float32, device="cuda")
        tq.tq_decode_attention_noalloc(gpu.layout, q, lens, gpu.k_codes, gpu.k_scales, gpu.v_codes, gpu.v_scales,
                                       w.scale, out, status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert_close(out.cpu().numpy(), ref, ATOL, RTOL_L2, what="no-alloc decode")


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
