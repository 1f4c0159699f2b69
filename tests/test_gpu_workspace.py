"""GPU parity of the decode on short and ragged caches, and of its use of the workspace.

Through the C ABI, against the oracle: ragged batches with empty sequences and
CTAs that straddle sequences, called repeatedly on one workspace; a workspace
filled with arbitrary bytes before the call (the decode reads nothing it has
not written in the same call); a CUDA graph replayed several times with new
queries; short and long caches decoded in turn on one shared workspace.
"""
import numpy as np
import pytest
import torch

from compressed_domain_attention_b200 import synthetic as syn
from compressed_domain_attention_b200 import tq
from tests.parity_utils import GpuCache, OracleCache, assert_close

pytestmark = pytest.mark.gpu


def case(lens, Hkv, G, D, seed, cap):
    B = len(lens)
    w = syn.Workload(f"ws_b{B}_h{Hkv}x{G}_d{D}", B, Hkv * G, Hkv, D, list(lens), torch.bfloat16, seed,
                     max_seq=cap)
    t = syn.generate(w)
    gpu = GpuCache(B, w.capacity, Hkv, Hkv * G, D)
    orc = OracleCache(B, w.capacity, Hkv, D)
    for b in range(B):
        if lens[b]:
            gpu.append_seq(b, t.k[b].cuda(), t.v[b].cuda(), 0)
            orc.append_seq(b, t.k[b], t.v[b], 0)
    torch.cuda.synchronize()
    return w, t, gpu, orc


def decode_into(gpu, q, lens, scale, ws, out, status):
    L = gpu.layout
    tq.tq_decode_attention(L, q.contiguous(), torch.tensor(lens, dtype=torch.int32, device="cuda"), gpu.k_codes,
                           gpu.k_scales, gpu.v_codes, gpu.v_scales, scale, out, ws, status)


@pytest.mark.parametrize("D,Hkv,G", [(256, 1, 4), (128, 2, 4), (64, 1, 8), (32, 2, 1)])
def test_ragged_with_empty_sequences_repeated_calls(D, Hkv, G):
    lens = [0, 1, 37, 300, 0, 129, 64]
    w, t, gpu, orc = case(lens, Hkv, G, D, 11 + D, 300)
    ws = tq.alloc_workspace(gpu.layout)
    out = torch.full((len(lens), Hkv * G, D), float("nan"), dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for rep in range(3):  # repeated calls on one workspace
        out.fill_(float("nan"))
        decode_into(gpu, t.q.cuda(), lens, w.scale, ws, out, status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        ref, st = orc.decode(t.q, lens, w.scale)
        assert st == 0
        got = out.cpu().numpy()
        assert np.all(got[[0, 4]] == 0.0), "empty sequences give zero rows"
        assert_close(got, ref, what=f"ragged D{D} rep {rep}")


def test_arbitrary_workspace_bytes():
    lens = [200, 17, 256]
    w, t, gpu, orc = case(lens, 1, 4, 256, 5, 256)
    ref, _ = orc.decode(t.q, lens, w.scale)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    g = torch.Generator(device="cpu").manual_seed(3)
    for fill in ("ones", "random"):
        ws = tq.alloc_workspace(gpu.layout)
        if fill == "ones":
            ws.fill_(0xFF)
        else:
            ws.copy_(torch.randint(0, 256, ws.shape, dtype=torch.uint8, generator=g).cuda())
        out = torch.full((3, 4, 256), float("nan"), dtype=torch.float32, device="cuda")
        decode_into(gpu, t.q.cuda(), lens, w.scale, ws, out, status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert_close(out.cpu().numpy(), ref, what=f"workspace of {fill}")


def test_graph_replays_with_new_queries():
    lens = [128, 300, 5]
    w, t, gpu, orc = case(lens, 2, 4, 128, 21, 300)
    ws = tq.alloc_workspace(gpu.layout)
    q = t.q.clone().cuda()
    out = torch.empty((3, 8, 128), dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    lens_d = torch.tensor(lens, dtype=torch.int32, device="cuda")
    decode_into(gpu, q, lens, w.scale, ws, out, status)  # warm-up outside the capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        tq.tq_decode_attention(gpu.layout, q, lens_d, gpu.k_codes, gpu.k_scales, gpu.v_codes, gpu.v_scales,
                               w.scale, out, ws, status, torch.cuda.current_stream())
    g = torch.Generator(device="cpu").manual_seed(9)
    for rep in range(4):
        qn = torch.randn(t.q.shape, generator=g).to(t.q.dtype)
        q.copy_(qn.cuda())
        graph.replay()
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        ref, _ = orc.decode(qn, lens, w.scale)
        assert_close(out.cpu().numpy(), ref, what=f"graph replay {rep}")
    del graph


def test_short_and_long_caches_share_one_workspace():
    # a short cache, then a long one and the short one again, sharing one workspace
    short = case([60, 250], 2, 4, 128, 31, 256)
    long_ = case([6000, 4096], 2, 4, 128, 32, 6000)
    ws = tq.alloc_workspace(long_[2].layout)
    assert ws.numel() >= short[2].layout.decode_workspace_bytes
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for w, t, gpu, orc in (short, long_, short):
        out = torch.empty((2, 8, 128), dtype=torch.float32, device="cuda")
        decode_into(gpu, t.q.cuda(), w.seq_lens, w.scale, ws, out, status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        ref, _ = orc.decode(t.q, w.seq_lens, w.scale)
        assert_close(out.cpu().numpy(), ref, what=w.name)
