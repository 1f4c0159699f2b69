"""Pins for the CPU oracle, independent of the oracle's own code.

Each test checks the oracle against something other than itself: a library
routine (scipy's Sylvester Hadamard matrix, torch's IEEE fp32->fp16 conversion),
a closed form, an exact invariant, brute force on tiny inputs, or an
original-domain fp64 attention computed here with numpy.

Page references (by title and section):
 * "Open-TQ-Metal: Fused Compressed-Domain Attention for Long-Context LLM
   Inference on Apple Silicon", abstract (cards page): sign-randomised
   transform + per-group abs-max + int4 nibble pack.
 * the same paper's arXiv abstract: attention directly on the compressed
   representation; 1/sqrt(d) attention scale.
 * mlxcel user guide "TurboQuant KV cache compression", §"What TurboQuant
   changes": Walsh-Hadamard rotation before low-bit storage.
 * "TurboQuant on AMD GPUs", §4: Walsh-Hadamard spreads energy evenly.
"""
import numpy as np
import pytest
import scipy.linalg
import torch

DIMS = (32, 64, 128, 256)


# ---------------------------------------------------------------- helpers (independent of the oracle)

def hadamard(D):
    return scipy.linalg.hadamard(D).astype(np.float64)  # Sylvester construction, natural order


def np_unpack(packed, D):
    lo = (packed & 0x0F).astype(np.int16)
    hi = (packed >> 4).astype(np.int16)
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    out = np.empty(packed.shape[:-1] + (D,), np.int16)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return out


def np_dequant_rotated(packed, scale_bits, D):
    codes = np_unpack(packed, D).astype(np.float64)
    sig = scale_bits.view(np.float16).astype(np.float64)
    return codes * np.repeat(sig, 32, axis=-1)


def np_dequant_original(packed, scale_bits, signs):
    D = signs.shape[0]
    y = np_dequant_rotated(packed, scale_bits, D)
    return (y @ hadamard(D).T) / np.sqrt(D) * signs.astype(np.float64)


def heavy_tailed(rng, n, D):
    x = rng.standard_normal((n, D)) * np.exp(rng.standard_normal(D))
    x[:, rng.permutation(D)[: D // 32]] *= 10.0
    return x.astype(np.float32)


# ---------------------------------------------------------------- sign vector / generator

def test_splitmix64_published_sequence(orc):
    # SplitMix64 (Vigna's public-domain reference generator), seed 0: the
    # widely reproduced first outputs.
    got = [int(x) for x in orc.splitmix64(0, 4)]
    assert got == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F, 0xF88BB8A8724C81EC]


def test_sign_vector_pm1_and_seeded(orc):
    for D in DIMS:
        s = orc.sign_vector(0, D)
        assert set(np.unique(s)) <= {-1.0, 1.0}
        assert np.array_equal(s, orc.sign_vector(0, D))
        r = orc.splitmix64(0, D)
        assert np.array_equal(s < 0, (r >> np.uint64(63)) == 1)
    assert not np.array_equal(orc.sign_vector(0, 128), orc.sign_vector(1, 128))
    # prefix property: the first 64 signs of the D=128 vector are the D=64 vector
    assert np.array_equal(orc.sign_vector(7, 128)[:64], orc.sign_vector(7, 64))


def test_norm_const(orc):
    assert orc.norm_const(64) == np.float32(0.125)
    assert orc.norm_const(256) == np.float32(0.0625)
    for D in (32, 128):
        c = float(orc.norm_const(D))
        # the binary32 nearest to 1/sqrt(D): within half an ulp of the exact value
        ulp = np.spacing(np.float32(c))
        assert abs(c - 1.0 / np.sqrt(D)) <= 0.5 * float(ulp)


# ---------------------------------------------------------------- Walsh-Hadamard transform

@pytest.mark.parametrize("D", DIMS)
def test_fwht_equals_sylvester_matrix(orc, D):
    # FWHT of the identity rows is H (exact: entries are sums of +-1).
    H = orc.fwht(np.eye(D, dtype=np.float32))
    assert np.array_equal(H.astype(np.float64), hadamard(D))
    # H H^T = D I exactly, via the oracle's transform applied to H's rows
    HH = orc.fwht(H)
    assert np.array_equal(HH, D * np.eye(D, dtype=np.float32))


@pytest.mark.parametrize("D", DIMS)
def test_fwht_matches_fp64_matrix_product(orc, D):
    rng = np.random.default_rng(D)
    x = rng.standard_normal((64, D)).astype(np.float32)
    got = orc.fwht(x).astype(np.float64)
    ref = x.astype(np.float64) @ hadamard(D).T
    scale = np.abs(x).sum(axis=1, keepdims=True)
    assert np.max(np.abs(got - ref) / scale) < 1e-6


@pytest.mark.parametrize("D", DIMS)
def test_srht_orthonormal_inverse_parseval(orc, D):
    s = orc.sign_vector(3, D)
    R = orc.srht_forward(np.eye(D, dtype=np.float32), s).astype(np.float64)  # row j = R e_j
    # rows of the forward image of the identity: R^T R = I
    assert np.max(np.abs(R @ R.T - np.eye(D))) < 1e-6
    # the map is c_D H diag(s)
    ref = (hadamard(D) * s.astype(np.float64)[None, :]).T / np.sqrt(D)
    assert np.max(np.abs(R - ref)) < 1e-7
    rng = np.random.default_rng(D + 1)
    x = heavy_tailed(rng, 32, D)
    y = orc.srht_forward(x, s)
    xb = orc.srht_inverse(y, s)
    assert np.max(np.abs(xb - x) / np.abs(x).max(axis=1, keepdims=True)) < 1e-6
    nx = np.linalg.norm(x.astype(np.float64), axis=1)
    ny = np.linalg.norm(y.astype(np.float64), axis=1)
    assert np.max(np.abs(ny / nx - 1)) < 1e-6


@pytest.mark.parametrize("D", DIMS)
def test_rotated_dot_products_equal_originals(orc, D):
    s = orc.sign_vector(0, D)
    rng = np.random.default_rng(10 + D)
    x = heavy_tailed(rng, 50, D)
    z = rng.standard_normal((50, D)).astype(np.float32)
    rx, rz = orc.srht_forward(x, s).astype(np.float64), orc.srht_forward(z, s).astype(np.float64)
    d0 = np.sum(x.astype(np.float64) * z, axis=1)
    d1 = np.sum(rx * rz, axis=1)
    bound = 1e-5 * np.linalg.norm(x, axis=1) * np.linalg.norm(z, axis=1)
    assert np.all(np.abs(d1 - d0) <= bound)


# ---------------------------------------------------------------- closed forms of the encoder

@pytest.mark.parametrize("D", DIMS)
def test_closed_form_unit_vector(orc, D):
    s = orc.sign_vector(5, D)
    H = hadamard(D)
    c = np.float32(1.0 / np.sqrt(D))
    sig16 = (np.float32(c) / np.float32(7.0)).astype(np.float16).view(np.uint16)
    for j in (0, 1, D // 2 - 1, D - 1):
        x = np.zeros(D, np.float32)
        x[j] = 1.0
        packed, scales, st = orc.encode(x[None], s)
        assert st == 0
        codes = np_unpack(packed[0], D)
        assert np.all(scales[0] == sig16)
        assert np.array_equal(codes, (7 * s[j] * H[:, j]).astype(np.int16))


@pytest.mark.parametrize("D", DIMS)
def test_closed_form_hadamard_column(orc, D):
    # x = s o H[:, j]  ->  y = fl(c_D * D) e_j exactly; one nonzero code (+7)
    s = orc.sign_vector(9, D)
    H = hadamard(D)
    for j in (0, 3, D - 1):
        x = (s.astype(np.float64) * H[:, j]).astype(np.float32)
        y = orc.srht_forward(x[None], s)[0]
        e = np.zeros(D, np.float32)
        e[j] = np.float32(D) * np.float32(1.0 / np.sqrt(D))
        assert np.array_equal(y, e)
        packed, scales, st = orc.encode(x[None], s)
        codes = np_unpack(packed[0], D)
        expect = np.zeros(D, np.int16)
        expect[j] = 7
        assert np.array_equal(codes, expect)
        g = j // 32
        sig = (e[j] / np.float32(7.0)).astype(np.float16).view(np.uint16)
        assert scales[0, g] == sig
        assert np.all(np.delete(scales[0], g) == 0)


# ---------------------------------------------------------------- quantiser

def brute_force_codes(y, sig):
    """argmin over c in [-7, 7] of |fl(y/sigma) - c|, ties to the even c."""
    r = (y / sig).astype(np.float32).astype(np.float64)
    cands = np.arange(-7, 8, dtype=np.float64)
    dist = np.abs(r[..., None] - cands)
    best = dist.min(axis=-1, keepdims=True)
    tie_even = np.where((dist == best) & (cands % 2 == 0), 0, 1) + np.where(dist == best, 0, 2)
    return cands[np.argmin(tie_even, axis=-1)].astype(np.int8)


@pytest.mark.parametrize("D", DIMS)
def test_quantiser_against_brute_force(orc, D):
    rng = np.random.default_rng(100 + D)
    y = heavy_tailed(rng, 400, D)
    # exact ties: absmax 7 gives sigma = 1, so y/sigma = k + 0.5 exactly
    y[0, :32] = np.concatenate([np.arange(-7.0, 7.5, 0.5), [0.25, -0.75, 6.75]]).astype(np.float32)
    codes, scales, st = orc.quantize_rotated(y)
    assert st == 0
    g = y.reshape(400, D // 32, 32)
    a = np.abs(g).max(axis=-1)
    sig16 = (a.astype(np.float32) / np.float32(7.0)).astype(np.float16)
    assert np.array_equal(scales, sig16.view(np.uint16))
    sig = sig16.astype(np.float32)[..., None]
    bf = np.where(sig > 0, brute_force_codes(g, np.where(sig > 0, sig, 1)), 0)
    assert np.array_equal(codes.reshape(bf.shape), bf)
    err = np.abs(g.astype(np.float64) - codes.reshape(g.shape) * sig.astype(np.float64))
    assert np.all(err <= sig.astype(np.float64) * (0.5 + 1e-6))
    assert codes.min() >= -7 and codes.max() <= 7


def test_quantiser_symmetries(orc):
    rng = np.random.default_rng(7)
    y = heavy_tailed(rng, 200, 128)
    c0, s0, _ = orc.quantize_rotated(y)
    c1, s1, _ = orc.quantize_rotated(-y)
    assert np.array_equal(c1, -c0) and np.array_equal(s1, s0)
    for k in (-3, 1, 4):
        c2, s2, _ = orc.quantize_rotated(np.ldexp(y, k))
        assert np.array_equal(c2, c0)
        assert np.array_equal(s2.view(np.float16).astype(np.float64),
                              np.ldexp(s0.view(np.float16).astype(np.float64), k))


def test_quantiser_zero_and_nonfinite_groups(orc):
    y = np.zeros((3, 64), np.float32)
    y[1, 3] = np.inf
    y[2, 40] = np.float32(1e6)  # absmax/7 overflows binary16
    codes, scales, st = orc.quantize_rotated(y)
    assert st & orc.STATUS_NONFINITE
    assert np.all(codes[0] == 0) and np.all(scales[0] == 0)
    assert scales[1, 0] == 0x7C00 and np.all(codes[1, :32] == 0) and scales[1, 1] == 0
    assert scales[2, 1] == 0x7C00 and np.all(codes[2, 32:] == 0)
    _, _, st0 = orc.quantize_rotated(np.ones((1, 64), np.float32))
    assert st0 == 0


# ---------------------------------------------------------------- binary16 conversion

@pytest.mark.slow
def test_f32_to_f16_exhaustive_against_torch(orc):
    # torch's float32->float16 cast is IEEE round-to-nearest-even (F16C on x86).
    n = 1 << 26
    for c in range((1 << 32) // n):
        bits = np.arange(c * n, (c + 1) * n, dtype=np.uint64).astype(np.uint32)
        x = bits.view(np.float32)
        got = orc.f32_to_f16_bits(x)
        ref = torch.from_numpy(x).to(torch.float16).view(torch.int16).numpy().view(np.uint16)
        nan = np.isnan(x)
        assert np.array_equal(got[~nan], ref[~nan]), hex(c * n)
        assert np.all((got[nan] & 0x7C00) == 0x7C00) and np.all((got[nan] & 0x3FF) != 0)


def test_f16_to_f32_exhaustive(orc):
    h = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    got = orc.f16_bits_to_f32(h)
    ref = h.view(np.float16).astype(np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(got.view(np.uint32)[~nan], ref.view(np.uint32)[~nan])
    assert np.all(np.isnan(got[nan]))


# ---------------------------------------------------------------- nibble packing

def test_pack_unpack_identity(orc):
    vals = np.arange(-7, 8, dtype=np.int8)
    pairs = np.array(np.meshgrid(vals, vals, indexing="ij")).reshape(2, -1).T  # 225 pairs
    flat = np.concatenate([pairs.reshape(-1), np.zeros(32 - pairs.size % 32, np.int8)]).reshape(-1, 32)
    packed = orc.pack(flat)
    assert np.array_equal(orc.unpack(packed, 32), flat)
    assert np.array_equal(np_unpack(packed, 32), flat)
    # every byte decodes, and re-encodes to itself (including the unused -8 nibble)
    allb = np.arange(256, dtype=np.uint16).astype(np.uint8).reshape(-1, 16)
    assert np.array_equal(orc.pack(orc.unpack(allb, 32)), allb)
    # low nibble = even element, two's complement
    one = np.zeros((1, 32), np.int8)
    one[0, 0], one[0, 1] = 3, -2
    assert orc.pack(one)[0, 0] == (3 | (0xE << 4))


# ---------------------------------------------------------------- rotation helps (motivation check)

def test_rotation_lowers_int4_roundtrip_error(orc):
    # [AMD] §4 / [MLX]: the Walsh-Hadamard rotation spreads outlier-channel
    # energy, so per-group abs-max wastes fewer levels.
    rng = np.random.default_rng(11)
    x = heavy_tailed(rng, 512, 128)
    s = orc.sign_vector(0, 128)
    packed, scales, _ = orc.encode(x, s)
    xr = np_dequant_original(packed, scales, s)
    c, sc, _ = orc.quantize_rotated(x)
    xn = c.astype(np.float64) * np.repeat(sc.view(np.float16).astype(np.float64), 32, axis=-1)
    mse_rot = np.mean((xr - x) ** 2)
    mse_plain = np.mean((xn - x) ** 2)
    assert mse_rot < 0.7 * mse_plain


# ---------------------------------------------------------------- attention

def make_cache(orc, rng, B, T, Hkv, D, s, max_seq=None, k=None, v=None):
    max_seq = max_seq or T
    if k is None:
        k = np.stack([heavy_tailed(rng, T * Hkv, D).reshape(T, Hkv, D) for _ in range(B)])
        v = rng.standard_normal((B, T, Hkv, D)).astype(np.float32)
    kc, ks = orc.new_cache(B, max_seq, Hkv, D)
    vc, vs = orc.new_cache(B, max_seq, Hkv, D)
    st = orc.quantize_append(s, k, v, np.zeros(B, np.int32), kc, ks, vc, vs)
    assert st == 0
    return kc, ks, vc, vs


def brute_force_attention(q, lens, kc, ks, vc, vs, s, sm_scale):
    """softmax(q K^T * scale) V in fp64 in the ORIGINAL domain on dequantised K, V."""
    B, Hq, D = q.shape
    Hkv = kc.shape[2]
    G = Hq // Hkv
    out = np.zeros((B, Hq, D))
    for b in range(B):
        L = lens[b]
        if L == 0:
            continue
        for hq in range(Hq):
            kv = hq // G
            K = np_dequant_original(kc[b, :L, kv], ks[b, :L, kv], s)
            V = np_dequant_original(vc[b, :L, kv], vs[b, :L, kv], s)
            z = K @ q[b, hq].astype(np.float64) * sm_scale
            w = np.exp(z - z.max())
            out[b, hq] = (w / w.sum()) @ V
    return out


@pytest.mark.parametrize("D,Hq,Hkv,T", [(32, 4, 1, 17), (128, 4, 1, 64), (128, 8, 2, 33), (64, 2, 2, 5),
                                        (256, 4, 1, 40)])
def test_attention_equals_fp64_original_domain(orc, D, Hq, Hkv, T):
    rng = np.random.default_rng(D * 1000 + T)
    s = orc.sign_vector(0, D)
    B = 2
    kc, ks, vc, vs = make_cache(orc, rng, B, T, Hkv, D, s)
    q = rng.standard_normal((B, Hq, D)).astype(np.float32)
    lens = np.array([T, max(1, T // 2)], np.int32)
    scale = 1.0 / np.sqrt(D)
    got, st = orc.decode_attention(s, q, lens, kc, ks, vc, vs, scale)
    assert st == 0
    ref = brute_force_attention(q, lens, kc, ks, vc, vs, s, scale)
    assert np.max(np.abs(got - ref)) < 2e-6 * max(1.0, np.abs(ref).max())


def test_attention_special_cases(orc):
    rng = np.random.default_rng(42)
    D, Hkv, Hq, T = 128, 2, 4, 24
    s = orc.sign_vector(0, D)
    kc, ks, vc, vs = make_cache(orc, rng, 1, T, Hkv, D, s)
    q = rng.standard_normal((1, Hq, D)).astype(np.float32)
    # T = 1: output = the one dequantised V row (original domain)
    out1, _ = orc.decode_attention(s, q, np.array([1], np.int32), kc, ks, vc, vs, 0.1)
    for hq in range(Hq):
        ref = np_dequant_original(vc[0, 0, hq // 2], vs[0, 0, hq // 2], s)
        assert np.max(np.abs(out1[0, hq] - ref)) < 1e-6 * max(1, np.abs(ref).max())
    # q = 0: uniform weights -> mean of dequantised V
    out0, _ = orc.decode_attention(s, np.zeros_like(q), np.array([T], np.int32), kc, ks, vc, vs, 0.1)
    for hq in range(Hq):
        ref = np_dequant_original(vc[0, :T, hq // 2], vs[0, :T, hq // 2], s).mean(axis=0)
        assert np.max(np.abs(out0[0, hq] - ref)) < 1e-6
    # all K rows identical -> mean of V for any q
    kc2, ks2 = kc.copy(), ks.copy()
    kc2[0, :] = kc[0, 0]
    ks2[0, :] = ks[0, 0]
    outk, _ = orc.decode_attention(s, q, np.array([T], np.int32), kc2, ks2, vc, vs, 0.3)
    assert np.max(np.abs(outk - out0)) < 1e-6
    # empty sequence -> zeros
    oute, st = orc.decode_attention(s, q, np.array([0], np.int32), kc, ks, vc, vs, 0.1)
    assert st == 0 and np.all(oute == 0)
    # length past max_seq -> capacity status, zeros
    outc, st = orc.decode_attention(s, q, np.array([T + 1], np.int32), kc, ks, vc, vs, 0.1)
    assert st & orc.STATUS_CAPACITY and np.all(outc == 0)


def test_gqa_equals_replicated_mha(orc):
    rng = np.random.default_rng(5)
    D, Hkv, G, T = 64, 2, 3, 19
    s = orc.sign_vector(0, D)
    k = np.stack([heavy_tailed(rng, T * Hkv, D).reshape(T, Hkv, D)])
    v = rng.standard_normal((1, T, Hkv, D)).astype(np.float32)
    kc, ks, vc, vs = make_cache(orc, rng, 1, T, Hkv, D, s, k=k, v=v)
    kr = np.repeat(k, G, axis=2)
    vr = np.repeat(v, G, axis=2)
    kc2, ks2, vc2, vs2 = make_cache(orc, rng, 1, T, Hkv * G, D, s, k=kr, v=vr)
    q = rng.standard_normal((1, Hkv * G, D)).astype(np.float32)
    lens = np.array([T], np.int32)
    a, _ = orc.decode_attention(s, q, lens, kc, ks, vc, vs, 0.125)
    b, _ = orc.decode_attention(s, q, lens, kc2, ks2, vc2, vs2, 0.125)
    assert np.array_equal(a, b)


def test_append_positions_and_capacity(orc):
    rng = np.random.default_rng(9)
    D, Hkv, S = 64, 2, 8
    s = orc.sign_vector(0, D)
    k = rng.standard_normal((2, 3, Hkv, D)).astype(np.float32)
    v = rng.standard_normal((2, 3, Hkv, D)).astype(np.float32)
    kc, ks = orc.new_cache(2, S, Hkv, D)
    vc, vs = orc.new_cache(2, S, Hkv, D)
    st = orc.quantize_append(s, k, v, np.array([2, 6], np.int32), kc, ks, vc, vs)
    assert st & orc.STATUS_CAPACITY  # 6 + 3 > 8: sequence 1 skipped
    p, sc, _ = orc.encode(k[0], s)
    assert np.array_equal(kc[0, 2:5], p) and np.array_equal(ks[0, 2:5], sc)
    assert np.all(kc[0, :2] == 0) and np.all(kc[0, 5:] == 0) and np.all(kc[1] == 0)
    pv, scv, _ = orc.encode(v[0], s)
    assert np.array_equal(vc[0, 2:5], pv) and np.array_equal(vs[0, 2:5], scv)


def test_dequantize_matches_independent(orc):
    rng = np.random.default_rng(12)
    D, Hkv, T = 128, 2, 10
    s = orc.sign_vector(0, D)
    kc, ks, _, _ = make_cache(orc, rng, 1, T, Hkv, D, s, max_seq=12)
    lens = np.array([T], np.int32)
    yr, _ = orc.dequantize(s, kc, ks, lens, False)
    xo, _ = orc.dequantize(s, kc, ks, lens, True)
    assert np.array_equal(yr[0, :T].astype(np.float64), np_dequant_rotated(kc[0, :T], ks[0, :T], D))
    assert np.max(np.abs(xo[0, :T] - np_dequant_original(kc[0, :T], ks[0, :T], s))) < 1e-5
    assert np.all(yr[0, T:] == 0) and np.all(xo[0, T:] == 0)


# ---------------------------------------------------------------- asymmetric cache (binary16 K, int4 V)
# mlxcel "TurboQuant KV cache compression", §"Cache modes": the recommended
# default keeps K in FP16 and compresses only V.

def make_cache_kf16(orc, rng, B, T, Hkv, D, s, k=None, v=None):
    if k is None:
        k = np.stack([heavy_tailed(rng, T * Hkv, D).reshape(T, Hkv, D) for _ in range(B)])
        v = rng.standard_normal((B, T, Hkv, D)).astype(np.float32)
    k16 = orc.new_k16_cache(B, T, Hkv, D)
    vc, vs = orc.new_cache(B, T, Hkv, D)
    st = orc.quantize_append_kf16(s, k, v, np.zeros(B, np.int32), k16, vc, vs)
    return k, v, k16, vc, vs, st


@pytest.mark.parametrize("D", DIMS)
def test_kf16_append_stores_numpy_binary16_and_the_symmetric_v(orc, D):
    rng = np.random.default_rng(D + 7)
    s = orc.sign_vector(0, D)
    k, v, k16, vc, vs, st = make_cache_kf16(orc, rng, 2, 9, 2, D, s)
    assert st == 0
    # K: numpy's own float32 -> float16 conversion (round to nearest even), bit for bit
    assert np.array_equal(k16, k.astype(np.float16).view(np.uint16))
    # V: the same bytes and scales as the symmetric append
    kc2, ks2 = orc.new_cache(2, 9, 2, D)
    vc2, vs2 = orc.new_cache(2, 9, 2, D)
    orc.quantize_append(s, k, v, np.zeros(2, np.int32), kc2, ks2, vc2, vs2)
    assert np.array_equal(vc, vc2) and np.array_equal(vs, vs2)


def test_kf16_append_overflow_and_capacity(orc):
    D = 32
    s = orc.sign_vector(0, D)
    k = np.zeros((1, 1, 1, D), np.float32)
    k[0, 0, 0, 3] = 70000.0  # beyond the binary16 range -> inf
    v = np.ones((1, 1, 1, D), np.float32)
    k16 = orc.new_k16_cache(1, 1, 1, D)
    vc, vs = orc.new_cache(1, 1, 1, D)
    st = orc.quantize_append_kf16(s, k, v, np.zeros(1, np.int32), k16, vc, vs)
    assert st & orc.STATUS_NONFINITE
    assert k16[0, 0, 0, 3] == 0x7C00
    st = orc.quantize_append_kf16(s, k, v, np.ones(1, np.int32), k16, vc, vs)  # position 1 of a 1-token cache
    assert st & orc.STATUS_CAPACITY


def brute_force_attention_kf16(q, lens, k16, vc, vs, s, sm_scale):
    """softmax(q K^T * scale) V in fp64: K the binary16 values, V dequantised to the original domain."""
    B, Hq, D = q.shape
    Hkv = vc.shape[2]
    G = Hq // Hkv
    out = np.zeros((B, Hq, D))
    for b in range(B):
        L = lens[b]
        if L == 0:
            continue
        for hq in range(Hq):
            kv = hq // G
            K = k16[b, :L, kv].view(np.float16).astype(np.float64)
            V = np_dequant_original(vc[b, :L, kv], vs[b, :L, kv], s)
            z = K @ q[b, hq].astype(np.float64) * sm_scale
            w = np.exp(z - z.max())
            out[b, hq] = (w / w.sum()) @ V
    return out


@pytest.mark.parametrize("D,Hq,Hkv,T", [(32, 4, 1, 17), (128, 4, 1, 64), (128, 16, 2, 33), (64, 2, 2, 5),
                                        (256, 4, 1, 40)])
def test_kf16_attention_equals_fp64_original_domain(orc, D, Hq, Hkv, T):
    rng = np.random.default_rng(D * 1000 + T + 1)
    s = orc.sign_vector(0, D)
    B = 2
    _, _, k16, vc, vs, st = make_cache_kf16(orc, rng, B, T, Hkv, D, s)
    assert st == 0
    q = rng.standard_normal((B, Hq, D)).astype(np.float32)
    lens = np.array([T, max(1, T // 2)], np.int32)
    scale = 1.0 / np.sqrt(D)
    got, st = orc.decode_attention_kf16(s, q, lens, k16, vc, vs, scale)
    assert st == 0
    ref = brute_force_attention_kf16(q, lens, k16, vc, vs, s, scale)
    assert np.max(np.abs(got - ref)) < 2e-6 * max(1.0, np.abs(ref).max())


def test_kf16_attention_special_cases(orc):
    rng = np.random.default_rng(43)
    D, Hkv, Hq, T = 128, 2, 4, 24
    s = orc.sign_vector(0, D)
    _, _, k16, vc, vs, _ = make_cache_kf16(orc, rng, 1, T, Hkv, D, s)
    q = rng.standard_normal((1, Hq, D)).astype(np.float32)
    # T = 1: the one dequantised V row (original domain)
    out1, _ = orc.decode_attention_kf16(s, q, np.array([1], np.int32), k16, vc, vs, 0.1)
    for hq in range(Hq):
        ref = np_dequant_original(vc[0, 0, hq // 2], vs[0, 0, hq // 2], s)
        assert np.max(np.abs(out1[0, hq] - ref)) < 1e-6 * max(1, np.abs(ref).max())
    # all K rows identical: uniform weights for any q -> mean of V; equals q = 0
    k2 = k16.copy()
    k2[0, :] = k16[0, 0]
    outk, _ = orc.decode_attention_kf16(s, q, np.array([T], np.int32), k2, vc, vs, 0.3)
    out0, _ = orc.decode_attention_kf16(s, np.zeros_like(q), np.array([T], np.int32), k16, vc, vs, 0.3)
    assert np.max(np.abs(outk - out0)) < 1e-6
    for hq in range(Hq):
        ref = np_dequant_original(vc[0, :T, hq // 2], vs[0, :T, hq // 2], s).mean(axis=0)
        assert np.max(np.abs(out0[0, hq] - ref)) < 1e-6
    # empty sequence and a length past max_seq
    oute, st = orc.decode_attention_kf16(s, q, np.array([0], np.int32), k16, vc, vs, 0.1)
    assert st == 0 and np.all(oute == 0)
    outc, st = orc.decode_attention_kf16(s, q, np.array([T + 1], np.int32), k16, vc, vs, 0.1)
    assert st & orc.STATUS_CAPACITY and np.all(outc == 0)


# ---------------------------------------------------------------- delegated hot/cold cache
# mlxcel "TurboQuant KV cache compression", §"Cache modes" (turbo4-delegated: K in
# FP16, V as an FP16 hot tail plus a 4-bit cold body) and §"Delegated cache variant".

# cold_length(len) for W = 8, F = 4 and W = 6, F = 3, worked by hand from the
# reading "at most W hot tokens, folded F at a time, oldest first"
COLD_W8_F4 = [0] * 9 + [4] * 4 + [8] * 4 + [12] * 4          # len 0..20
COLD_W6_F3 = [0] * 7 + [3] * 3 + [6] * 3 + [9] * 3           # len 0..15


def test_delegated_cold_length_worked_values_and_invariants(orc):
    assert [orc.cold_length(n, 8, 4) for n in range(21)] == COLD_W8_F4
    assert [orc.cold_length(n, 6, 3) for n in range(16)] == COLD_W6_F3
    for W, F in ((1, 1), (16, 16), (64, 16), (256, 64), (100, 7)):
        prev = 0
        for n in range(0, 5 * W + 3):
            c = orc.cold_length(n, W, F)
            assert c % F == 0 and c >= prev and c - prev in (0, F)
            hot = n - c
            assert (hot == n) if n <= W else (W - F < hot <= W)
            prev = c


def make_delegated(orc, s, k, v, W, F, chunks=None, max_seq=None):
    """Append k, v [B][T][Hkv][D] into a fresh delegated cache, in one call or in the given chunk sizes."""
    B, T, Hkv, D = k.shape
    S = max_seq or T
    k16 = orc.new_k16_cache(B, S, Hkv, D)
    vc, vs = orc.new_cache(B, S, Hkv, D)
    tail = orc.new_tail(B, W, Hkv, D)
    st = 0
    pos = 0
    for c in (chunks or [T]):
        st |= orc.append_delegated(s, k[:, pos:pos + c], v[:, pos:pos + c], np.full(B, pos, np.int32), W, F,
                                   k16, vc, vs, tail)
        pos += c
    assert pos == T
    return k16, vc, vs, tail, st


@pytest.mark.parametrize("D,W,F,T", [(32, 8, 4, 21), (128, 8, 4, 13), (64, 6, 3, 6), (128, 16, 16, 40)])
def test_delegated_append_holds_binary16_tail_and_encoded_body(orc, D, W, F, T):
    rng = np.random.default_rng(D + W + T)
    s = orc.sign_vector(0, D)
    B, Hkv = 2, 2
    k = rng.standard_normal((B, T, Hkv, D)).astype(np.float32)
    v = np.stack([heavy_tailed(rng, T * Hkv, D).reshape(T, Hkv, D) for _ in range(B)])
    k16, vc, vs, tail, st = make_delegated(orc, s, k, v, W, F)
    assert st == 0
    # K: numpy's binary16 of every token
    assert np.array_equal(k16, k.astype(np.float16).view(np.uint16))
    nc = orc.cold_length(T, W, F)
    v16 = v.astype(np.float16)
    # hot tokens: numpy's binary16 of V, at slot t mod W
    for t in range(nc, T):
        assert np.array_equal(tail[:, t % W], v16[:, t].view(np.uint16))
    # cold tokens: the symmetric encoding of the binary16-rounded V, bit for bit
    kc2, ks2 = orc.new_cache(B, T, Hkv, D)
    vc2, vs2 = orc.new_cache(B, T, Hkv, D)
    orc.quantize_append(s, k, v16.astype(np.float32), np.zeros(B, np.int32), kc2, ks2, vc2, vs2)
    assert np.array_equal(vc[:, :nc], vc2[:, :nc]) and np.array_equal(vs[:, :nc], vs2[:, :nc])


def test_delegated_append_is_chunking_invariant(orc):
    rng = np.random.default_rng(99)
    D, W, F, T, B, Hkv = 64, 8, 4, 37, 2, 2
    s = orc.sign_vector(5, D)
    k = rng.standard_normal((B, T, Hkv, D)).astype(np.float32)
    v = rng.standard_normal((B, T, Hkv, D)).astype(np.float32)
    ref = make_delegated(orc, s, k, v, W, F)
    nc = orc.cold_length(T, W, F)
    live = sorted({t % W for t in range(nc, T)})
    for chunks in ([1] * T, [3, 9, 1, 1, 20, 3], [8, 8, 8, 8, 5], [30, 7]):
        got = make_delegated(orc, s, k, v, W, F, chunks)
        assert np.array_equal(got[0], ref[0])
        assert np.array_equal(got[1][:, :nc], ref[1][:, :nc]) and np.array_equal(got[2][:, :nc], ref[2][:, :nc])
        assert np.array_equal(got[3][:, live], ref[3][:, live])


def brute_force_attention_delegated(q, lens, k16, vc, vs, tail, s, W, F, cold_len, sm_scale):
    """softmax(q K^T * scale) V in fp64 with the cache's own values: binary16 K; V the dequantised
    original-domain body below cold_len(len), the binary16 tail value above."""
    B, Hq, D = q.shape
    Hkv = vc.shape[2]
    G = Hq // Hkv
    out = np.zeros((B, Hq, D))
    for b in range(B):
        L = lens[b]
        if L == 0:
            continue
        nc = cold_len(L)
        for hq in range(Hq):
            kv = hq // G
            K = k16[b, :L, kv].view(np.float16).astype(np.float64)
            V = np.empty((L, D))
            if nc:
                V[:nc] = np_dequant_original(vc[b, :nc, kv], vs[b, :nc, kv], s)
            for t in range(nc, L):
                V[t] = tail[b, t % W, kv].view(np.float16).astype(np.float64)
            z = K @ q[b, hq].astype(np.float64) * sm_scale
            w = np.exp(z - z.max())
            out[b, hq] = (w / w.sum()) @ V
    return out


@pytest.mark.parametrize("D,Hq,Hkv,W,F,T", [(32, 4, 1, 8, 4, 21), (128, 8, 1, 16, 8, 50), (64, 4, 2, 6, 3, 6),
                                            (128, 16, 2, 32, 32, 33)])
def test_delegated_attention_equals_fp64(orc, D, Hq, Hkv, W, F, T):
    rng = np.random.default_rng(D + Hq + W + T)
    s = orc.sign_vector(0, D)
    B = 3
    k = rng.standard_normal((B, T, Hkv, D)).astype(np.float32)
    v = rng.standard_normal((B, T, Hkv, D)).astype(np.float32)
    k16, vc, vs, tail, st = make_delegated(orc, s, k, v, W, F)
    assert st == 0
    q = rng.standard_normal((B, Hq, D)).astype(np.float32)
    scale = 1.0 / np.sqrt(D)
    # decode at the full length only: shorter lengths would read tail slots a later token overwrote
    lens = np.array([T, T, T], np.int32)
    got, st = orc.decode_attention_delegated(s, q, lens, k16, vc, vs, tail, W, F, scale)
    assert st == 0
    # cold_length restated from the worked tables' rule, not through the oracle
    cold = lambda n: 0 if n <= W else -(-(n - W) // F) * F
    ref = brute_force_attention_delegated(q, lens, k16, vc, vs, tail, s, W, F, cold, scale)
    assert np.max(np.abs(got - ref)) < 2e-6 * max(1.0, np.abs(ref).max())


def test_delegated_all_hot_is_binary16_attention_of_the_inputs(orc):
    # len <= W: nothing is quantised; the output is softmax attention over the
    # binary16-rounded inputs themselves (no cache values read here)
    rng = np.random.default_rng(7)
    D, Hq, Hkv, W, F, T, B = 128, 4, 1, 32, 8, 32, 1
    s = orc.sign_vector(0, D)
    k = rng.standard_normal((B, T, Hkv, D)).astype(np.float32)
    v = rng.standard_normal((B, T, Hkv, D)).astype(np.float32)
    k16, vc, vs, tail, _ = make_delegated(orc, s, k, v, W, F)
    q = rng.standard_normal((B, Hq, D)).astype(np.float32)
    for L in (1, 17, 32):
        got, _ = orc.decode_attention_delegated(s, q, np.array([L], np.int32), k16, vc, vs, tail, W, F, 0.2)
        K = k[0, :L, 0].astype(np.float16).astype(np.float64)
        V = v[0, :L, 0].astype(np.float16).astype(np.float64)
        for hq in range(Hq):
            z = K @ q[0, hq].astype(np.float64) * 0.2
            w = np.exp(z - z.max())
            ref = (w / w.sum()) @ V
            assert np.max(np.abs(got[0, hq] - ref)) < 1e-6


def test_delegated_special_cases(orc):
    rng = np.random.default_rng(3)
    D, W, F = 32, 4, 2
    s = orc.sign_vector(0, D)
    k = rng.standard_normal((1, 6, 1, D)).astype(np.float32)
    v = rng.standard_normal((1, 6, 1, D)).astype(np.float32)
    v[0, 5, 0, 1] = 1.0e5  # beyond binary16
    k16, vc, vs, tail, st = make_delegated(orc, s, k, v, W, F)
    assert st & orc.STATUS_NONFINITE
    assert tail[0, 5 % W, 0, 1] == 0x7C00
    q = rng.standard_normal((1, 2, D)).astype(np.float32)
    out, st = orc.decode_attention_delegated(s, q, np.array([0], np.int32), k16, vc, vs, tail, W, F, 0.1)
    assert st == 0 and np.all(out == 0)
    out, st = orc.decode_attention_delegated(s, q, np.array([7], np.int32), k16, vc, vs, tail, W, F, 0.1)
    assert st & orc.STATUS_CAPACITY and np.all(out == 0)
    st = orc.append_delegated(s, k[:, :1], v[:, :1], np.array([6], np.int32), W, F, k16, vc, vs, tail)
    assert st & orc.STATUS_CAPACITY


# ---------------------------------------------------------------- per-channel lambda and sparse-V
# Open-TQ-Metal abstract (the fused kernel's step list: transform, per-channel
# lambda, per-group abs-max, int4 pack); mlxcel guide §"Sparse-V dequant
# threshold" (skip V dequant where the attention weight is below 1e-6).

def test_lambda_sits_between_the_transform_and_the_abs_max(orc):
    rng = np.random.default_rng(17)
    D = 128
    s = orc.sign_vector(0, D)
    x = heavy_tailed(rng, 9, D)
    lam = np.exp(rng.uniform(-1, 1, D)).astype(np.float32)
    got_p, got_s, st = orc.encode_lambda(x, s, lam)
    assert st == 0
    # the definition restated: the pinned transform, one binary32 multiply per channel
    # (numpy's IEEE float32 product), then the pinned quantiser and packing
    y = orc.srht_forward(x, s) * lam
    codes, scales, _ = orc.quantize_rotated(y)
    assert np.array_equal(got_p, orc.pack(codes)) and np.array_equal(got_s, scales)
    # lambda = None and lambda = 1 are the plain encoder
    p0, s0, _ = orc.encode(x, s)
    p1, s1, _ = orc.encode_lambda(x, s, None)
    p2, s2, _ = orc.encode_lambda(x, s, np.ones(D, np.float32))
    assert np.array_equal(p0, p1) and np.array_equal(p0, p2) and np.array_equal(s0, s1) and np.array_equal(s0, s2)


def test_lambda_powers_of_two_per_group_keep_codes_and_shift_scales(orc):
    rng = np.random.default_rng(18)
    D = 128
    s = orc.sign_vector(0, D)
    x = rng.standard_normal((7, D)).astype(np.float32)
    e = np.array([-3, 0, 2, 5])  # one exponent per group of 32
    lam = np.repeat(np.exp2(e), 32).astype(np.float32)
    p_l, s_l, _ = orc.encode_lambda(x, s, lam)
    p_0, s_0, _ = orc.encode(x, s)
    assert np.array_equal(p_l, p_0)  # y * 2^e and sigma * 2^e: the same quotients
    want = (s_0.view(np.float16).astype(np.float64) * np.exp2(e)).astype(np.float16).view(np.uint16)
    assert np.array_equal(s_l, want)


def np_dequant_original_lambda(packed, scale_bits, signs, lam):
    D = signs.shape[0]
    y = np_dequant_rotated(packed, scale_bits, D)
    if lam is not None:
        y = y / lam.astype(np.float64)
    return (y @ hadamard(D).T) / np.sqrt(D) * signs.astype(np.float64)


def make_cache_lambda(orc, rng, B, T, Hkv, D, s, lk, lv):
    k = np.stack([heavy_tailed(rng, T * Hkv, D).reshape(T, Hkv, D) for _ in range(B)])
    v = rng.standard_normal((B, T, Hkv, D)).astype(np.float32)
    kc, ks = orc.new_cache(B, T, Hkv, D)
    vc, vs = orc.new_cache(B, T, Hkv, D)
    st = orc.quantize_append_lambda(s, k, v, np.zeros(B, np.int32), lk, lv, kc, ks, vc, vs)
    assert st == 0
    return kc, ks, vc, vs


def brute_force_ext(q, lens, kc, ks, vc, vs, s, scale, lk=None, lv=None, tau=0.0):
    """fp64 attention over the dequantised cache (lambda undone), dropping the V term of tokens
    with exp(z - max z) < tau; also the bound sum_dropped w |V|."""
    B, Hq, D = q.shape
    Hkv = vc.shape[2]
    G = Hq // Hkv
    out = np.zeros((B, Hq, D))
    bound = np.zeros((B, Hq, D))
    for b in range(B):
        L = lens[b]
        if L == 0:
            continue
        for hq in range(Hq):
            kv = hq // G
            K = np_dequant_original_lambda(kc[b, :L, kv], ks[b, :L, kv], s, lk)
            V = np_dequant_original_lambda(vc[b, :L, kv], vs[b, :L, kv], s, lv)
            z = K @ q[b, hq].astype(np.float64) * scale
            r = np.exp(z - z.max())
            w = r / r.sum()
            keep = ~(r < tau) if tau > 0 else np.ones(L, bool)
            out[b, hq] = w[keep] @ V[keep]
            bound[b, hq] = w[~keep] @ np.abs(V[~keep]) if (~keep).any() else 0.0
    return out, bound


@pytest.mark.parametrize("D,Hq,Hkv,T", [(128, 8, 2, 40), (64, 4, 1, 33), (32, 2, 2, 17)])
def test_lambda_attention_equals_fp64(orc, D, Hq, Hkv, T):
    rng = np.random.default_rng(D + Hq + T)
    s = orc.sign_vector(3, D)
    lk = np.exp(rng.uniform(-1, 1, D)).astype(np.float32)
    lv = np.exp(rng.uniform(-1, 1, D)).astype(np.float32)
    kc, ks, vc, vs = make_cache_lambda(orc, rng, 2, T, Hkv, D, s, lk, lv)
    q = rng.standard_normal((2, Hq, D)).astype(np.float32)
    lens = np.array([T, T // 2], np.int32)
    got, bound, st = orc.decode_attention_ext(s, q, lens, kc, ks, vc, vs, 0.2, lk, lv)
    assert st == 0 and np.all(bound == 0)
    ref, _ = brute_force_ext(q, lens, kc, ks, vc, vs, s, 0.2, lk, lv)
    assert np.max(np.abs(got - ref)) < 2e-6 * max(1.0, np.abs(ref).max())


def test_sparse_v_zero_threshold_is_exact_and_the_drop_rule(orc):
    rng = np.random.default_rng(21)
    D, Hq, Hkv, T, B = 128, 8, 2, 300, 2
    s = orc.sign_vector(0, D)
    kc, ks, vc, vs = make_cache_lambda(orc, rng, B, T, Hkv, D, s, None, None)
    q = (4.0 * rng.standard_normal((B, Hq, D))).astype(np.float32)  # peaked weights
    lens = np.array([T, 200], np.int32)
    exact, _ = orc.decode_attention(s, q, lens, kc, ks, vc, vs, 0.3)
    got0, b0, _ = orc.decode_attention_ext(s, q, lens, kc, ks, vc, vs, 0.3, tau=0.0)
    assert np.array_equal(got0, exact) and np.all(b0 == 0)
    for tau in (1e-6, 1e-3, 0.5):
        got, bound, st = orc.decode_attention_ext(s, q, lens, kc, ks, vc, vs, 0.3, tau=tau)
        ref, rb = brute_force_ext(q, lens, kc, ks, vc, vs, s, 0.3, tau=tau)
        assert st == 0
        assert np.max(np.abs(got - ref)) < 2e-6 * max(1.0, np.abs(ref).max())
        assert np.max(np.abs(bound - rb)) < 2e-5 * max(1.0, rb.max())  # binary32 inverse transform per token
        # the bound covers the change from exact attention
        assert np.all(np.abs(got.astype(np.float64) - exact) <= bound + 1e-5)
    assert rb.max() > 0  # tau = 0.5 drops tokens here
    # near-uniform weights: each normalised weight is about 1/T, each relative weight about 1,
    # so a threshold between the two separates "relative to the largest score" from "normalised"
    qd = (0.05 * rng.standard_normal((B, Hq, D))).astype(np.float32)
    got, bound, _ = orc.decode_attention_ext(s, qd, lens, kc, ks, vc, vs, 0.3, tau=0.01)
    ref, rb = brute_force_ext(qd, lens, kc, ks, vc, vs, s, 0.3, tau=0.01)
    assert np.max(np.abs(got - ref)) < 2e-6 * max(1.0, np.abs(ref).max())


# ---------------------------------------------------------------- paged storage
# mlxcel guide, §"Known limitations / paged KV scheduler": a paged decode storage
# backend. A paged cache is the contiguous cache with its rows moved to pool pages.

def paged_table(rng, B, max_seq, P, n_pages):
    max_pages = -(-max_seq // P)
    perm = rng.permutation(n_pages)[: B * max_pages]
    return perm.reshape(B, max_pages).astype(np.int32)


@pytest.mark.parametrize("kf16", [False, True])
def test_paged_cache_is_the_contiguous_cache_with_rows_moved(orc, kf16):
    rng = np.random.default_rng(61 + kf16)
    B, T, Hkv, D, P = 3, 45, 2, 64, 16
    n_pages = B * (-(-T // P)) + 5
    s = orc.sign_vector(0, D)
    k = rng.standard_normal((B, T, Hkv, D)).astype(np.float32)
    v = rng.standard_normal((B, T, Hkv, D)).astype(np.float32)
    table = paged_table(rng, B, T, P, n_pages)
    pools = orc.new_pool(n_pages, P, Hkv, D, kf16)
    # in chunks that cross page boundaries
    pos = 0
    for c in (7, 16, 1, 21):
        st = orc.quantize_append_paged(s, k[:, pos:pos + c], v[:, pos:pos + c], np.full(B, pos, np.int32), table,
                                       P, T, pools)
        assert st == 0
        pos += c
    # the pinned contiguous append of the same tokens
    vc, vs = orc.new_cache(B, T, Hkv, D)
    if kf16:
        kc = orc.new_k16_cache(B, T, Hkv, D)
        orc.quantize_append_kf16(s, k, v, np.zeros(B, np.int32), kc, vc, vs)
    else:
        kc, ks = orc.new_cache(B, T, Hkv, D)
        orc.quantize_append(s, k, v, np.zeros(B, np.int32), kc, ks, vc, vs)
    pk, pks, pv, pvs = pools
    for b in range(B):
        for t in range(T):
            r = table[b, t // P] * P + t % P
            assert np.array_equal(pk[r], kc[b, t]) and np.array_equal(pv[r], vc[b, t]) and np.array_equal(pvs[r], vs[b, t])
            if not kf16:
                assert np.array_equal(pks[r], ks[b, t])
    # decode: the same values as the contiguous decode
    q = rng.standard_normal((B, 4, D)).astype(np.float32)
    lens = np.array([T, 17, 0], np.int32)
    got, st = orc.decode_attention_paged(s, q, lens, table, P, T, pools, 0.15)
    if kf16:
        ref, _ = orc.decode_attention_kf16(s, q, lens, kc, vc, vs, 0.15)
    else:
        ref, _ = orc.decode_attention(s, q, lens, kc, ks, vc, vs, 0.15)
    assert st == 0 and np.array_equal(got, ref)


def test_paged_unmapped_page_is_skipped_with_status(orc):
    rng = np.random.default_rng(63)
    B, T, Hkv, D, P = 1, 40, 1, 32, 16
    s = orc.sign_vector(0, D)
    table = np.array([[2, -1, 0]], np.int32)
    pools = orc.new_pool(3, P, Hkv, D)
    k = rng.standard_normal((B, T, Hkv, D)).astype(np.float32)
    st = orc.quantize_append_paged(s, k, k, np.zeros(B, np.int32), table, P, T, pools)
    assert st & orc.STATUS_CAPACITY
    assert np.all(pools[2][1 * P:2 * P] == 0)  # page 1 was never mapped, so never written
    assert np.any(pools[2][2 * P:3 * P] != 0) and np.any(pools[2][0:P] != 0)
