"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI
and the CPU oracle on the same seeded inputs, and compare."""
import numpy as np
import torch

import oracle
from compressed_domain_attention_b200 import tq

ATOL = 2e-3     # decode tolerance: max-abs error vs the oracle's fp32 result
RTOL_L2 = 1e-3  # and relative L2 error


def np_f32(t):
    return t.detach().to("cpu", torch.float32).contiguous().numpy()


class GpuCache:
    """A packed K/V cache in device memory laid out by tq_cache_layout."""

    def __init__(self, batch, max_seq, n_kv, n_q, D, sign_seed=0, device="cuda", k_format=tq.TQ_K_INT4):
        self.layout = tq.tq_cache_layout_kv(batch, max_seq, n_kv, n_q, D, k_format, 32, sign_seed)
        self.k_codes, self.k_scales, self.v_codes, self.v_scales = tq.alloc_cache(self.layout, device)
        self.device = device
        self.kf16 = k_format == tq.TQ_K_FP16

    def seq_view(self, b):
        """(layout, k_codes, k_scales, v_codes, v_scales) for sequence b alone (a batch-1 view)."""
        L = self.layout
        l1 = tq.tq_cache_layout_kv(1, L.max_seq, L.n_kv_heads, L.n_q_heads, L.head_dim, L.k_format, 32, L.sign_seed)
        cs, ss, ks_ = int(L.code_stride_seq), int(L.scale_stride_seq), int(L.k_stride_seq)
        return (l1, self.k_codes[b * ks_:(b + 1) * ks_], None if self.kf16 else self.k_scales[b * ss:],
                self.v_codes[b * cs:(b + 1) * cs], self.v_scales[b * ss:])

    def append_seq(self, b, k, v, start, status=None):
        """Append k, v [n][Hkv][D] to sequence b at position start."""
        l1, kc, ks, vc, vs = self.seq_view(b)
        sp = torch.tensor([start], dtype=torch.int32, device=self.device)
        tq.tq_quantize_append(l1, k[None].contiguous(), v[None].contiguous(), k.shape[0], sp, kc, ks, vc, vs, status)

    def append_all(self, k, v, start_pos, status=None):
        """k, v [B][n][Hkv][D]; start_pos int list."""
        sp = torch.tensor(start_pos, dtype=torch.int32, device=self.device)
        tq.tq_quantize_append(self.layout, k.contiguous(), v.contiguous(), k.shape[1], sp, self.k_codes,
                              self.k_scales, self.v_codes, self.v_scales, status)

    def host_arrays(self):
        """(k_codes, k_scales, v_codes, v_scales) as numpy [B][S][Hkv][...] (scales as uint16 bits)."""
        L = self.layout
        B, S, H, D = L.batch, L.max_seq, L.n_kv_heads, L.head_dim
        n_s = B * S * H * (D // 32)
        vc = self.v_codes.cpu().numpy().reshape(B, S, H, D // 2)
        if self.kf16:  # binary16 K bits [B][S][H][D], no K scales
            kc = self.k_codes.cpu().numpy().view(np.uint16).reshape(B, S, H, D)
            ks = None
        else:
            kc = self.k_codes.cpu().numpy().reshape(B, S, H, D // 2)
            ks = self.k_scales[:n_s].cpu().numpy().view(np.uint16).reshape(B, S, H, D // 32)
        vs = self.v_scales[:n_s].cpu().numpy().view(np.uint16).reshape(B, S, H, D // 32)
        return kc, ks, vc, vs

    def decode(self, q, seq_lens, sm_scale, status=None, **opts):
        L = self.layout
        out = torch.full((L.batch, L.n_q_heads, L.head_dim), float("nan"), dtype=torch.float32, device=self.device)
        ws = tq.alloc_workspace(L, self.device)
        lens = torch.tensor(seq_lens, dtype=torch.int32, device=self.device)
        tq.tq_decode_attention(L, q.contiguous(), lens, self.k_codes, self.k_scales, self.v_codes, self.v_scales,
                               sm_scale, out, ws, status, **opts)
        return out


class OracleCache:
    def __init__(self, batch, max_seq, n_kv, D, sign_seed=0, kf16=False):
        self.signs = oracle.sign_vector(sign_seed, D)
        self.kf16 = kf16
        if kf16:
            self.kc, self.ks = oracle.new_k16_cache(batch, max_seq, n_kv, D), None
        else:
            self.kc, self.ks = oracle.new_cache(batch, max_seq, n_kv, D)
        self.vc, self.vs = oracle.new_cache(batch, max_seq, n_kv, D)

    def append_seq(self, b, k, v, start):
        sp = np.array([start], np.int32)
        if self.kf16:
            st = oracle.quantize_append_kf16(self.signs, np_f32(k)[None], np_f32(v)[None], sp, self.kc[b:b + 1],
                                             self.vc[b:b + 1], self.vs[b:b + 1])
        else:
            st = oracle.quantize_append(self.signs, np_f32(k)[None], np_f32(v)[None], sp, self.kc[b:b + 1],
                                        self.ks[b:b + 1], self.vc[b:b + 1], self.vs[b:b + 1])
        assert st == 0

    def decode(self, q, seq_lens, sm_scale, which=None):
        lens = np.asarray(seq_lens, np.int32)
        if self.kf16:
            return oracle.decode_attention_kf16(self.signs, np_f32(q), lens, self.kc, self.vc, self.vs, sm_scale,
                                                which)
        out, st = oracle.decode_attention(self.signs, np_f32(q), lens, self.kc, self.ks, self.vc, self.vs, sm_scale,
                                          which)
        return out, st


def assert_close(got, ref, atol=ATOL, rtol_l2=RTOL_L2, what=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    max_abs = float(err.max()) if err.size else 0.0
    rel = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30))
    assert max_abs <= atol and rel <= rtol_l2, f"{what}: max_abs {max_abs:.3e} (<= {atol}), rel_l2 {rel:.3e} (<= {rtol_l2})"
    return max_abs, rel
