"""Pins of the fp64 oracle: checks against things other than the oracle itself.

Each ``pin_*`` takes a loaded oracle library and raises AssertionError on a
mismatch.  They are run against the committed oracle (test_oracle_pins.py)
and against deliberately broken copies of it (test_oracle_mutants.py), which
shows that a plausible slip anywhere in the oracle fails at least one pin.

What pins what:
  * half decoding       -> numpy's float16 -> float64 conversion, all 65536 patterns;
  * memory formula      -> the pages' worked 70B example (tests/golden);
  * attention core      -> torch's scaled_dot_product_attention in float64 on a
                           contiguous cache (a textbook routine), identity table;
  * the gather          -> bit-identical results under a permuted placement, and
                           a pure-Python brute force through a permuted table;
  * GQA grouping        -> SDPA with each KV head repeated over its query group;
  * causal verify       -> SDPA with an explicit causal mask, and row j equal to a
                           decode over the first L - q_len + j + 1 tokens;
  * closed forms        -> one token gives V; q = 0 gives the mean of V; a key that
                           dominates by far gives its V;
  * append / block copy -> numpy slot views of the pool.
"""
from __future__ import annotations

import math

import numpy as np
import torch
import torch.nn.functional as F

import oracle
from conftest import read_golden


def _rng(seed):
    return np.random.Generator(np.random.PCG64(seed))


def _f16(rng, shape, scale=1.0):
    return (rng.standard_normal(shape) * scale).astype(np.float16)


def _contiguous_to_pool(kc, bs):
    """[Hkv][L][D] contiguous cache -> identity-placed pool [nb][Hkv][bs][D]."""
    Hkv, L, D = kc.shape
    nb = -(-L // bs)
    pad = np.zeros((Hkv, nb * bs, D), dtype=kc.dtype)
    pad[:, :L] = kc
    return np.ascontiguousarray(pad.reshape(Hkv, nb, bs, D).transpose(1, 0, 2, 3))


def _sdpa(q, k, v, scale, mask=None):
    """q [Hq][n][D], k/v [Hq][L][D] (float64) -> [Hq][n][D]."""
    return F.scaled_dot_product_attention(torch.from_numpy(q), torch.from_numpy(k),
                                          torch.from_numpy(v), attn_mask=mask,
                                          scale=scale).numpy()


def pin_half_decoding(L):
    pats = np.arange(65536, dtype=np.uint16)
    ref = pats.view(np.float16).astype(np.float64)
    got = np.array([L.oracle_half_to_double(int(p)) for p in pats[::7]])
    ref = ref[::7]
    both_nan = np.isnan(ref) & np.isnan(got)
    assert np.array_equal(got[~both_nan], ref[~both_nan])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    for p in (0x0001, 0x03FF, 0x0400, 0x3C00, 0x7BFF, 0x7C00, 0xFC00, 0x8001, 0xC000):
        r = np.array([p], dtype=np.uint16).view(np.float16).astype(np.float64)[0]
        assert L.oracle_half_to_double(p) == r


def pin_memory_formula(L):
    rows, _ = read_golden("kv_memory_formula.txt")
    for layers, heads, hd, seq, batch, dt, gib in rows:
        b = L.oracle_kv_cache_bytes(int(layers), int(heads), int(hd), int(seq), int(batch),
                                    int(dt))
        assert b == float(gib) * 2**30, (b, gib)
    # pool form: capacity in tokens replaces seq_len x batch, KV heads replace heads
    assert (L.oracle_pool_bytes_per_layer(1000, 16, 8, 128, 2)
            == L.oracle_kv_cache_bytes(1, 8, 128, 16000, 1, 2) == 2 * 8 * 128 * 16000 * 2)


def _case(seed, B, Hq, Hkv, D, bs, lens, q_len=1):
    rng = _rng(seed)
    G = Hq // Hkv
    q = _f16(rng, (B, q_len, Hq, D))
    kc = [_f16(rng, (Hkv, int(n), D)) for n in lens]
    vc = [_f16(rng, (Hkv, int(n), D)) for n in lens]
    return rng, G, q, kc, vc


def _pack(kc_list, vc_list, bs, perm_seed=None):
    """Place several contiguous caches into one pool; identity order unless
    perm_seed is given, in which case physical ids are permuted."""
    pools_k = [_contiguous_to_pool(k, bs) for k in kc_list]
    pools_v = [_contiguous_to_pool(v, bs) for v in vc_list]
    nbs = [p.shape[0] for p in pools_k]
    total = sum(nbs)
    Kp = np.concatenate(pools_k)
    Vp = np.concatenate(pools_v)
    ids = np.arange(total)
    if perm_seed is not None:
        perm = _rng(perm_seed).permutation(total)
        K2 = np.empty_like(Kp)
        V2 = np.empty_like(Vp)
        K2[perm] = Kp
        V2[perm] = Vp
        Kp, Vp, ids = K2, V2, perm
    tables = np.full((len(nbs), max(nbs)), -1, dtype=np.int32)
    off = 0
    for s, n in enumerate(nbs):
        tables[s, :n] = ids[off:off + n]
        off += n
    return Kp, Vp, tables


def pin_attention_vs_sdpa(L):
    for seed, (Hq, Hkv, D, bs, lens) in enumerate([(4, 4, 16, 4, [1, 7, 13]),
                                                   (8, 2, 32, 8, [9, 24, 3]),
                                                   (6, 3, 8, 16, [33, 16])]):
        B = len(lens)
        rng, G, q, kc, vc = _case(100 + seed, B, Hq, Hkv, D, bs, lens)
        Kp, Vp, tables = _pack(kc, vc, bs)
        scale = 1.0 / math.sqrt(D)
        got = oracle.paged_attention(q, Kp, Vp, tables, np.array(lens, np.int32), scale=scale,
                                     L=L)
        for s in range(B):
            k = np.repeat(kc[s].astype(np.float64), G, axis=0)  # [Hq][L][D]
            v = np.repeat(vc[s].astype(np.float64), G, axis=0)
            ref = _sdpa(q[s, 0].astype(np.float64)[:, None, :], k, v, scale)[:, 0, :]
            np.testing.assert_allclose(got[s, 0], ref, rtol=1e-12, atol=1e-12)


def pin_permutation_invariance(L):
    lens = [5, 21, 40, 16]
    rng, G, q, kc, vc = _case(7, 4, 4, 2, 16, 8, lens)
    a = _pack(kc, vc, 8)
    b = _pack(kc, vc, 8, perm_seed=11)
    assert not np.array_equal(a[2], b[2])
    cl = np.array(lens, np.int32)
    oa = oracle.paged_attention(q, a[0], a[1], a[2], cl, scale=0.25, L=L)
    ob = oracle.paged_attention(q, b[0], b[1], b[2], cl, scale=0.25, L=L)
    assert np.array_equal(oa, ob)


def pin_brute_force(L):
    """Pure-Python definition through a permuted table (tiny sizes)."""
    lens = [3, 6]
    B, Hq, Hkv, D, bs = 2, 4, 2, 4, 4
    rng, G, q, kc, vc = _case(5, B, Hq, Hkv, D, bs, lens)
    Kp, Vp, tables = _pack(kc, vc, bs, perm_seed=3)
    scale = 0.7
    got = oracle.paged_attention(q, Kp, Vp, tables, np.array(lens, np.int32), scale=scale, L=L)
    for s in range(B):
        for h in range(Hq):
            g = h // G
            sc = []
            for t in range(lens[s]):
                blk = int(tables[s][t // bs])
                sc.append(scale * sum(float(q[s, 0, h, d]) * float(Kp[blk, g, t % bs, d])
                                      for d in range(D)))
            m = max(sc)
            w = [math.exp(x - m) for x in sc]
            z = sum(w)
            for d in range(D):
                ref = sum(w[t] * float(Vp[int(tables[s][t // bs]), g, t % bs, d])
                          for t in range(lens[s])) / z
                assert abs(got[s, 0, h, d] - ref) <= 1e-12 * max(1.0, abs(ref))


def pin_verify_causal(L):
    lens = [12, 30]
    q_len, Hq, Hkv, D, bs = 5, 4, 2, 16, 8
    rng, G, q, kc, vc = _case(9, 2, Hq, Hkv, D, bs, lens, q_len=q_len)
    Kp, Vp, tables = _pack(kc, vc, bs, perm_seed=2)
    cl = np.array(lens, np.int32)
    got = oracle.paged_attention(q, Kp, Vp, tables, cl, scale=0.3, q_len=q_len, L=L)
    for s in range(2):
        n = lens[s]
        k = np.repeat(kc[s].astype(np.float64), G, axis=0)
        v = np.repeat(vc[s].astype(np.float64), G, axis=0)
        qq = q[s].astype(np.float64).transpose(1, 0, 2)  # [Hq][q_len][D]
        j = np.arange(q_len)[:, None]
        t = np.arange(n)[None, :]
        mask = torch.from_numpy(t <= (n - q_len + j))
        ref = _sdpa(qq, k, v, 0.3, mask=mask).transpose(1, 0, 2)
        np.testing.assert_allclose(got[s], ref, rtol=1e-12, atol=1e-12)
        # row j equals a plain decode over the first n - q_len + j + 1 tokens
        for jj in range(q_len):
            one = oracle.paged_attention(np.ascontiguousarray(q[s:s + 1, jj:jj + 1]), Kp, Vp,
                                         tables[s:s + 1],
                                         np.array([n - q_len + jj + 1], np.int32),
                                         scale=0.3, L=L)
            assert np.array_equal(one[0, 0], got[s, jj])


def pin_closed_forms(L):
    D, bs, Hkv = 8, 4, 1
    rng = _rng(21)
    # single token -> exactly V
    q = _f16(rng, (1, 1, 1, D))
    k = _f16(rng, (1, 1, D))
    v = _f16(rng, (1, 1, D))
    Kp, Vp, tb = _pack([k], [v], bs, perm_seed=1)
    out = oracle.paged_attention(q, Kp, Vp, tb, np.array([1], np.int32), scale=1.0, L=L)
    assert np.array_equal(out[0, 0, 0], v[0, 0].astype(np.float64))
    # q = 0 -> mean of V (equal weights)
    n = 11
    k = _f16(rng, (1, n, D))
    v = _f16(rng, (1, n, D))
    Kp, Vp, tb = _pack([k], [v], bs, perm_seed=4)
    out = oracle.paged_attention(np.zeros((1, 1, 1, D), np.float16), Kp, Vp, tb,
                                 np.array([n], np.int32), scale=0.5, L=L)
    np.testing.assert_allclose(out[0, 0, 0], v[0].astype(np.float64).mean(0), rtol=1e-13,
                               atol=1e-15)
    # one key dominates by exp(-400): output is that key's V
    qd = np.zeros((1, 1, 1, D), np.float16)
    qd[..., 0] = 1.0
    k = np.zeros((1, n, D), np.float16)
    k[0, 6, 0] = 400.0
    out = oracle.paged_attention(qd, *_pack([k], [v], bs, perm_seed=5), np.array([n], np.int32),
                                 scale=1.0, L=L)
    assert np.array_equal(out[0, 0, 0], v[0, 6].astype(np.float64))
    # empty context -> zeros
    out = oracle.paged_attention(qd, Kp, Vp, tb, np.array([0], np.int32), scale=1.0, L=L)
    assert not out.any()


def pin_shared_prefix_equals_private(L):
    """Tables sharing physical prefix blocks give what private copies give."""
    rng = _rng(31)
    Hkv, D, bs = 2, 8, 4
    pre = 8  # two full blocks
    kpre, vpre = _f16(rng, (Hkv, pre, D)), _f16(rng, (Hkv, pre, D))
    suf = [3, 6]
    ks = [np.concatenate([kpre, _f16(rng, (Hkv, n, D))], 1) for n in suf]
    vs = [np.concatenate([vpre, _f16(rng, (Hkv, n, D))], 1) for n in suf]
    Kp, Vp, tables = _pack(ks, vs, bs)  # private copies of the prefix
    shared = tables.copy()
    shared[1, :2] = shared[0, :2]       # second table points at the first's prefix
    Kp2, Vp2 = Kp.copy(), Vp.copy()
    Kp2[tables[1, :2]] = np.nan         # the private prefix copy is now garbage
    Vp2[tables[1, :2]] = np.nan
    q = _f16(rng, (2, 1, 4, D))
    cl = np.array([pre + n for n in suf], np.int32)
    a = oracle.paged_attention(q, Kp, Vp, tables, cl, scale=0.4, L=L)
    b = oracle.paged_attention(q, Kp2, Vp2, shared, cl, scale=0.4, L=L)
    assert np.array_equal(a, b)


def pin_append(L):
    rng = _rng(41)
    nb, Hkv, bs, D, T = 6, 3, 4, 8, 5
    K = _f16(rng, (nb, Hkv, bs, D))
    V = _f16(rng, (nb, Hkv, bs, D))
    kn = _f16(rng, (T, Hkv, D))
    vn = _f16(rng, (T, Hkv, D))
    slots = np.array([0, 23, -1, 10, 13], np.int64)
    K2, V2 = oracle.append(K, V, kn, vn, slots, L=L)
    # slot view of a pool: [Hkv][nb*bs][D]
    view = lambda P: P.transpose(1, 0, 2, 3).reshape(Hkv, nb * bs, D)
    refK, refV = view(K).copy(), view(V).copy()
    for t, sl in enumerate(slots):
        if sl >= 0:
            refK[:, sl] = kn[t]
            refV[:, sl] = vn[t]
    assert np.array_equal(view(K2).view(np.uint16), refK.view(np.uint16))
    assert np.array_equal(view(V2).view(np.uint16), refV.view(np.uint16))
    try:
        oracle.append(K, V, kn, vn, np.array([0, 1, 2, 3, nb * bs], np.int64), L=L)
        raise AssertionError("slot beyond the pool was accepted")
    except ValueError:
        pass


def pin_copy_blocks(L):
    rng = _rng(51)
    nb, Hkv, bs, D = 7, 2, 4, 8
    K = _f16(rng, (nb, Hkv, bs, D))
    V = _f16(rng, (nb, Hkv, bs, D))
    K2, V2 = oracle.copy_blocks(K, V, np.array([[1, 4], [6, 0]], np.int32), L=L)
    refK, refV = K.copy(), V.copy()
    refK[4], refV[4] = K[1], V[1]
    refK[0], refV[0] = K[6], V[6]
    assert np.array_equal(K2.view(np.uint16), refK.view(np.uint16))
    assert np.array_equal(V2.view(np.uint16), refV.view(np.uint16))


def pin_q8k_attention_exact_scales(L):
    """Power-of-two scales make every dequantised key an fp16 value: attention
    over the codes must equal the fp16 attention on those values bit for bit
    (scale factor, its (head, channel) index, code pool layout)."""
    rng = _rng(61)
    nb, Hkv, bs, D, Hq = 12, 2, 4, 16, 4
    codes = rng.integers(-128, 128, size=(nb, Hkv, bs, D)).astype(np.int8)
    scales = np.ldexp(1.0, -rng.integers(3, 9, size=(Hkv, D))).astype(np.float32)
    exact = codes.astype(np.float64) * scales[None, :, None, :].astype(np.float64)
    kdq = exact.astype(np.float16)
    assert np.array_equal(kdq.astype(np.float64), exact)
    V = _f16(rng, (nb, Hkv, bs, D))
    lens = np.array([13, 20, 1], np.int32)
    perm = rng.permutation(nb).astype(np.int32)
    tables = np.full((3, 5), -1, np.int32)
    tables[0, :4], tables[1, :5], tables[2, :1] = perm[:4], perm[4:9], perm[9:10]
    q = _f16(rng, (3, 1, Hq, D))
    got = oracle.paged_attention_q8k(q, codes, scales, V, tables, lens, scale=0.25, L=L)
    ref = oracle.paged_attention(q, kdq, V, tables, lens, scale=0.25, L=L)
    assert np.array_equal(got, ref)


def pin_q8k_codes(L):
    """Scales and codes: the channel maximum maps to +-127, the round trip
    stays within half a step, codes are odd in k, exact half steps round to
    even and clamp at the ends, and codes land where the fp16 append puts K."""
    rng = _rng(71)
    T, Hkv, D = 40, 3, 8
    k = _f16(rng, (T, Hkv, D), 2.0)
    k[:, 2, 5] = 0                                   # an all-zero channel
    sc = oracle.k_scales(k, L=L)
    assert sc.shape == (Hkv, D) and sc[2, 5] == 1.0
    kf = k.astype(np.float64)
    amax = np.abs(kf).max(axis=0)
    live = amax > 0
    # ~ max|k| / 127 (the step that spans the symmetric 8-bit range)
    np.testing.assert_allclose(sc[live], amax[live] / 127.0, rtol=1e-6)
    slots = np.arange(T, dtype=np.int64)
    zk = np.zeros((T, Hkv, 1, D), np.int8)
    zv = np.zeros((T, Hkv, 1, D), np.float16)
    K8, V2 = oracle.append_q8k(zk, zv, k, -k, slots, sc, L=L)
    c = K8[:, :, 0, :].astype(np.int64)
    assert np.array_equal(V2[:, :, 0, :].view(np.uint16), (-k).view(np.uint16))
    arg = np.abs(kf).argmax(axis=0)
    top = np.take_along_axis(c, arg[None], axis=0)[0]
    assert np.array_equal(top[live], np.sign(np.take_along_axis(kf, arg[None], axis=0)[0])[live] * 127)
    assert np.all(np.abs(c * sc.astype(np.float64)[None] - kf) <= sc.astype(np.float64)[None] * (0.5 + 1e-6))
    Kn, _ = oracle.append_q8k(zk, zv, -k, k, slots, sc, L=L)
    assert np.array_equal(Kn.astype(np.int64), -K8.astype(np.int64))
    # half steps with an exact scale of 1/4
    half = np.array([0.125, 0.375, -0.125, -0.375, 0.625, 31.875, -32.125, 33.0, -33.0,
                     np.inf, -np.inf, np.nan], np.float16)
    want = np.array([0, 2, 0, -2, 2, 127, -128, 127, -128, 127, -128, 0], np.int64)
    n = half.size
    hk = np.zeros((n, 1, D), np.float16)
    hk[:, 0, 3] = half
    s4 = np.full((1, D), 0.25, np.float32)
    H8, _ = oracle.append_q8k(np.zeros((n, 1, 1, D), np.int8), np.zeros((n, 1, 1, D), np.float16),
                              hk, hk, np.arange(n, dtype=np.int64), s4, L=L)
    assert np.array_equal(H8[:, 0, 0, 3].astype(np.int64), want)
    # placement: exact multiples of power-of-two scales go where the fp16
    # append puts them
    nb, bs = 5, 4
    p2 = np.ldexp(1.0, -rng.integers(2, 6, size=(Hkv, D))).astype(np.float32)
    cc = rng.integers(-127, 128, size=(7, Hkv, D))
    kk = (cc * p2[None].astype(np.float64)).astype(np.float16)
    sl = np.array([3, 17, -1, 0, 9, 12, 19], np.int64)
    Q8, _ = oracle.append_q8k(np.zeros((nb, Hkv, bs, D), np.int8), np.zeros((nb, Hkv, bs, D), np.float16),
                              kk, kk, sl, p2, L=L)
    F16, _ = oracle.append(np.zeros((nb, Hkv, bs, D), np.float16), np.zeros((nb, Hkv, bs, D), np.float16),
                           kk, kk, sl, L=L)
    assert np.array_equal(Q8.astype(np.float64) * p2[None, :, None, :], F16.astype(np.float64))


PINS = [pin_half_decoding, pin_memory_formula, pin_attention_vs_sdpa, pin_permutation_invariance,
        pin_brute_force, pin_verify_causal, pin_closed_forms, pin_shared_prefix_equals_private,
        pin_append, pin_copy_blocks, pin_q8k_attention_exact_scales, pin_q8k_codes]
