"""Failure detection on the GPU without a fault: bounded pipeline waits.

Every wait of the split-K decode kernel (for a tile's copies, its converted
scales, or a free stage) is bounded by the GPU's global timer. When one runs
out, the kernel sets TQ_STATUS_TIMEOUT in the caller's status word, stops
reading tiles, waits for the copies it already has in flight and returns, so
the context stays usable. Here a bound of a few nanoseconds makes the waits run
out on a multi-megabyte cache; nothing faults, traps or hangs. The call must
return (the stream synchronises), report the timeout, and the next call with
the default bound must match the oracle.
"""
import pytest
import torch

from compressed_domain_attention_b200 import synthetic as syn
from compressed_domain_attention_b200 import tq
from tests.parity_utils import GpuCache, OracleCache, assert_close

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("G,k_format", [(8, tq.TQ_K_INT4), (4, tq.TQ_K_INT4), (4, tq.TQ_K_FP16)])
def test_bounded_wait_runs_out_and_the_next_call_is_exact(G, k_format):
    T = 32768  # 8 kv heads: about 38 MB of int4 cache, several tiles per split-K block
    w = syn.Workload(f"timeout_g{G}", 1, 8 * G, 8, 128, [T], torch.bfloat16, 61)
    t = syn.generate(w)
    kf = k_format == tq.TQ_K_FP16
    gpu = GpuCache(1, T, 8, 8 * G, 128, k_format=k_format)
    gpu.append_seq(0, t.k[0].cuda(), t.v[0].cuda(), 0)
    orc = OracleCache(1, T, 8, 128, kf16=kf)
    orc.append_seq(0, t.k[0], t.v[0], 0)
    q = t.q.cuda()
    for _ in range(2):
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        gpu.decode(q, [T], w.scale, status, wait_limit_ns=2)
        torch.cuda.synchronize()  # the call returned: no block is left waiting
        assert int(status.item()) & tq.TQ_STATUS_TIMEOUT
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = gpu.decode(q, [T], w.scale, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref, st = orc.decode_all(t.q, [T], w.scale, G)
    assert st == 0
    assert_close(out.cpu().numpy(), ref, what=f"after a timeout, G{G}")


def test_wait_limit_rejects_negative_values():
    gpu = GpuCache(1, 64, 1, 4, 128)
    q = torch.zeros((1, 4, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(tq.TqError) as exc:
        gpu.decode(q, [8], 0.1, wait_limit_ns=-1)
    assert exc.value.code == tq.TQ_ERR_INVALID_ARG
