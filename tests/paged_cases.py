"""Test helpers: small paged cases built from contiguous K/V, and the
independent checks the oracle is pinned to.

Every case starts from contiguous per-sequence K and V and scatters them into
a NaN-filled pool through a random block table, so that the dense and
brute-force checks below never look at the paged layout.
"""
from __future__ import annotations

from decimal import Decimal, getcontext

import numpy as np
import scipy.special

from workloads import nan_bits, to_storage_bits


def widen_bits(bits: np.ndarray, dtype: str) -> np.ndarray:
    """uint16 patterns -> float64 via numpy's own fp16 / fp32 conversions."""
    bits = np.asarray(bits, dtype=np.uint16)
    if dtype == "f16":
        return bits.view(np.float16).astype(np.float64)
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def paged_case(rng, ctx_list, H, D, bs, num_blocks=None, dtype="f16", scale=None):
    """Contiguous K/V per sequence, scattered into a pool [NB, H, bs, D]."""
    ctx_list = [int(c) for c in ctx_list]
    S = len(ctx_list)
    nblk = [-(-c // bs) for c in ctx_list]
    need = sum(nblk)
    NB = num_blocks if num_blocks is not None else need + 3
    perm = rng.permutation(NB)
    nan = nan_bits(dtype)
    kpool = np.full((NB, H, bs, D), nan, dtype=np.uint16)
    vpool = np.full((NB, H, bs, D), nan, dtype=np.uint16)
    MB = max(1, max(nblk, default=1))
    bt = np.full((S, MB), -1, dtype=np.int32)
    K, V = [], []
    nxt = 0
    for s, c in enumerate(ctx_list):
        blocks = perm[nxt: nxt + nblk[s]]
        nxt += nblk[s]
        bt[s, : nblk[s]] = blocks
        k = to_storage_bits(rng.standard_normal((c, H, D), dtype=np.float32), dtype)
        v = to_storage_bits(rng.standard_normal((c, H, D), dtype=np.float32), dtype)
        if c:
            j = np.arange(c)
            kpool[blocks[j // bs], :, j % bs, :] = k
            vpool[blocks[j // bs], :, j % bs, :] = v
        K.append(k)
        V.append(v)
    q = to_storage_bits(rng.standard_normal((S, H, D), dtype=np.float32), dtype)
    if scale is None:
        scale = np.float32(1.0 / np.sqrt(D))
    return dict(q=q, K=K, V=V, kpool=kpool, vpool=vpool, bt=bt,
                ctx=np.array(ctx_list, dtype=np.int32), scale=np.float32(scale),
                dtype=dtype, bs=bs)


def dense_attention(q, K, V, scale, dtype="f16"):
    """softmax(scale q K^T) V on the unpaged copy, through scipy's softmax.
    q [H, D], K/V [n, H, D] as uint16 patterns; returns float64 [H, D]."""
    qf = widen_bits(q, dtype)
    if K.shape[0] == 0:
        return np.zeros_like(qf)
    Kf, Vf = widen_bits(K, dtype), widen_bits(V, dtype)
    scores = float(scale) * np.einsum("hd,nhd->hn", qf, Kf)
    p = scipy.special.softmax(scores, axis=-1)
    return np.einsum("hn,nhd->hd", p, Vf)


def brute_force(q, K, V, scale, dtype="f16", digits=50):
    """The same quantity in 50-digit decimal arithmetic, one (head) at a time.
    Returns float64 [H, D]."""
    getcontext().prec = digits
    qf, Kf, Vf = widen_bits(q, dtype), widen_bits(K, dtype), widen_bits(V, dtype)
    H, D = qf.shape
    n = Kf.shape[0]
    sc = Decimal(float(scale))
    out = np.zeros((H, D))
    for h in range(H):
        if n == 0:
            continue
        qd = [Decimal(float(x)) for x in qf[h]]
        s = []
        for j in range(n):
            s.append(sc * sum(qd[d] * Decimal(float(Kf[j, h, d])) for d in range(D)))
        m = max(s)
        w = [(x - m).exp() for x in s]
        z = sum(w)
        for d in range(D):
            out[h, d] = float(sum(w[j] * Decimal(float(Vf[j, h, d])) for j in range(n)) / z)
    return out


# ---------------------------------------------------------------------------
# Pins. Each takes an oracle.Oracle and raises AssertionError on a mismatch.
# ---------------------------------------------------------------------------

def _decode_case(orc, c):
    return orc.decode(c["q"], c["kpool"], c["vpool"], c["bt"], c["ctx"], c["scale"],
                      c["dtype"])


def pin_dense(orc, seed=11):
    rng = np.random.default_rng(seed)
    for H, D, bs, ctxs, dtype in [
        (2, 64, 16, [1, 15, 16, 17, 40], "f16"),
        (3, 128, 8, [7, 64, 100], "f16"),
        (2, 128, 32, [31, 33, 200], "f16"),
        (2, 64, 16, [5, 50], "bf16"),
    ]:
        c = paged_case(rng, ctxs, H, D, bs, dtype=dtype)
        got = _decode_case(orc, c)
        for s in range(len(ctxs)):
            ref = dense_attention(c["q"][s], c["K"][s], c["V"][s], c["scale"], dtype)
            err = np.max(np.abs(got[s] - ref))
            assert err <= 1e-12, f"dense mismatch {err} (H{H} D{D} bs{bs} s{s})"


def pin_bruteforce(orc, seed=12):
    rng = np.random.default_rng(seed)
    c = paged_case(rng, [1, 17, 33, 100], 4, 64, 16, scale=0.125)
    got = _decode_case(orc, c)
    for s in range(4):
        ref = brute_force(c["q"][s], c["K"][s], c["V"][s], c["scale"])
        err = np.max(np.abs(got[s] - ref))
        assert err <= 1e-12, f"brute-force mismatch {err} (seq {s})"


def pin_closed_forms(orc, seed=13):
    rng = np.random.default_rng(seed)
    H, D, bs = 2, 64, 16
    # ctx = 1: the output is the single value row, exactly.
    c = paged_case(rng, [1, 1], H, D, bs)
    got = _decode_case(orc, c)
    for s in range(2):
        assert np.array_equal(got[s], widen_bits(c["V"][s][0], "f16")), "ctx=1 != v0"
    # scale = 0: uniform weights, the output is the mean of the value rows.
    c = paged_case(rng, [37, 5], H, D, bs, scale=0.0)
    got = _decode_case(orc, c)
    for s in range(2):
        ref = widen_bits(c["V"][s], "f16").mean(axis=0)
        assert np.max(np.abs(got[s] - ref)) <= 1e-13, "scale=0 != mean(V)"
    # All keys equal: again the mean of the value rows.
    c = paged_case(rng, [23], H, D, bs)
    row = c["K"][0][0].copy()
    c["K"][0][:] = row
    j = np.arange(23)
    c["kpool"][c["bt"][0][j // bs], :, j % bs, :] = c["K"][0]
    got = _decode_case(orc, c)
    ref = widen_bits(c["V"][0], "f16").mean(axis=0)
    assert np.max(np.abs(got[0] - ref)) <= 1e-13, "equal keys != mean(V)"
    # Two tokens: o = (v0 + e^d v1) / (1 + e^d), d = scale (q.k1 - q.k0).
    c = paged_case(rng, [2], H, D, bs)
    qf = widen_bits(c["q"][0], "f16")
    kf, vf = widen_bits(c["K"][0], "f16"), widen_bits(c["V"][0], "f16")
    got = _decode_case(orc, c)
    for h in range(H):
        d = float(c["scale"]) * (qf[h] @ kf[1, h] - qf[h] @ kf[0, h])
        a = 1.0 / (1.0 + np.exp(d))
        ref = a * vf[0, h] + (1.0 - a) * vf[1, h]
        assert np.max(np.abs(got[0, h] - ref)) <= 1e-13, "two-token closed form"
    # One dominant token with scores in the thousands: the output is that
    # token's value row (and nothing overflows).
    c = paged_case(rng, [50], H, D, bs, scale=np.float32(64.0))
    k = widen_bits(c["K"][0], "f16")
    qf = widen_bits(c["q"][0], "f16")
    got = _decode_case(orc, c)
    checked = 0
    for h in range(H):
        sc = k[:, h] @ qf[h]
        top = np.argsort(sc)[-2:]
        assert np.all(np.isfinite(got[0, h])), "overflow with large scores"
        if 64.0 * (sc[top[1]] - sc[top[0]]) > 60:
            ref = widen_bits(c["V"][0][top[1], h], "f16")
            assert np.max(np.abs(got[0, h] - ref)) <= 1e-12, "dominant token"
            checked += 1
    assert checked >= 1, "no head had a dominant token; change the seed"


def pin_permutation(orc, seed=14):
    """Moving every physical block to another id (and the tables with it)
    leaves the output bit-identical."""
    rng = np.random.default_rng(seed)
    c = paged_case(rng, [3, 16, 41, 90], 3, 64, 16, num_blocks=24)
    got = _decode_case(orc, c)
    NB = c["kpool"].shape[0]
    pi = rng.permutation(NB)
    k2 = np.empty_like(c["kpool"])
    v2 = np.empty_like(c["vpool"])
    k2[pi] = c["kpool"]
    v2[pi] = c["vpool"]
    bt2 = np.where(c["bt"] >= 0, pi[np.maximum(c["bt"], 0)], -1).astype(np.int32)
    got2 = orc.decode(c["q"], k2, v2, bt2, c["ctx"], c["scale"])
    assert np.array_equal(got, got2), "not invariant under a block permutation"


def pin_write_kv(orc, seed=15):
    """Appending tokens one by one through slots fills a sequence so that the
    gathered cache equals the tokens written; nothing else changes."""
    rng = np.random.default_rng(seed)
    H, D, bs, NB = 2, 64, 8, 12
    nan = nan_bits("f16")
    kc = np.full((NB, H, bs, D), nan, dtype=np.uint16)
    vc = kc.copy()
    blocks = rng.permutation(NB)[:4]
    n = 29
    toks_k = to_storage_bits(rng.standard_normal((n, H, D), dtype=np.float32), "f16")
    toks_v = to_storage_bits(rng.standard_normal((n, H, D), dtype=np.float32), "f16")
    for t in range(n):  # one token per decode step, like the engine does
        slot = np.array([blocks[t // bs] * bs + t % bs], dtype=np.int64)
        orc.write_kv(toks_k[t:t + 1], toks_v[t:t + 1], slot, kc, vc, bs)
    for t in range(n):
        assert np.array_equal(kc[blocks[t // bs], :, t % bs, :], toks_k[t]), "K slot"
        assert np.array_equal(vc[blocks[t // bs], :, t % bs, :], toks_v[t]), "V slot"
    written = np.zeros((NB, bs), dtype=bool)
    for t in range(n):
        written[blocks[t // bs], t % bs] = True
    assert np.all(kc.transpose(0, 2, 1, 3)[~written] == nan), "K written elsewhere"
    assert np.all(vc.transpose(0, 2, 1, 3)[~written] == nan), "V written elsewhere"
    # A negative slot is padding: nothing is written.
    before = kc.copy()
    orc.write_kv(toks_k[:1], toks_v[:1], np.array([-1], dtype=np.int64), kc, vc, bs)
    assert np.array_equal(before, kc), "padding slot wrote"
    # The round trip through the oracle's own decode: a sequence whose K/V
    # went in through write_kv decodes like the dense copy.
    bt = np.full((1, 4), -1, dtype=np.int32)
    bt[0] = blocks
    q = to_storage_bits(rng.standard_normal((1, H, D), dtype=np.float32), "f16")
    got = orc.decode(q, kc, vc, bt, np.array([n], dtype=np.int32), np.float32(0.125))
    ref = dense_attention(q[0], toks_k, toks_v, np.float32(0.125))
    assert np.max(np.abs(got[0] - ref)) <= 1e-12, "write_kv round trip"


def pin_write_kv_batched(orc, seed=21):
    """Many tokens in one write call, padding slots among them (a batch of
    sequences appending at once, "vLLM基础", §2.2 steps 4-6): row t of the
    input lands at its own slot and nowhere else, checked against direct
    numpy placement; the fp8 write stores each row's codes and scale as the
    brute-force nearest-value encoding of that same row."""
    rng = np.random.default_rng(seed)
    H, D, bs, NB = 3, 64, 8, 10
    T = 13
    slots = rng.permutation(NB * bs)[:T].astype(np.int64)
    slots[[2, 7, 11]] = -1                      # padding rows
    nan = nan_bits("f16")
    keys = to_storage_bits(rng.standard_normal((T, H, D), dtype=np.float32), "f16")
    vals = to_storage_bits(rng.standard_normal((T, H, D), dtype=np.float32), "f16")
    kc = np.full((NB, H, bs, D), nan, dtype=np.uint16)
    vc = kc.copy()
    orc.write_kv(keys, vals, slots, kc, vc, bs)
    want_k = np.full_like(kc, nan)
    want_v = np.full_like(vc, nan)
    for t in range(T):
        if slots[t] >= 0:
            want_k[slots[t] // bs, :, slots[t] % bs, :] = keys[t]
            want_v[slots[t] // bs, :, slots[t] % bs, :] = vals[t]
    assert np.array_equal(kc, want_k), "batched K write differs from direct placement"
    assert np.array_equal(vc, want_v), "batched V write differs from direct placement"
    # The same batch into an fp8 pool.
    table = e4m3_table()
    tb = bs * D + 4 * bs
    kq = np.full((NB, H, tb), 0x7F, dtype=np.uint8)
    vq = kq.copy()
    orc.write_kv_fp8(keys, vals, slots, kq, vq, bs)
    written = np.zeros((NB, bs), dtype=bool)
    for t in range(T):
        if slots[t] < 0:
            continue
        b, o = slots[t] // bs, slots[t] % bs
        written[b, o] = True
        for h in range(H):
            for pool, raw in ((kq, keys), (vq, vals)):
                x = raw[t, h].view(np.float16).astype(np.float32)
                amax = np.float32(np.max(np.abs(x)))
                sc = pool[b, h, bs * D + 4 * o: bs * D + 4 * o + 4].view(np.float32)[0]
                assert sc == amax / np.float32(448.0), "batched fp8 row scale"
                codes = pool[b, h, o * D:(o + 1) * D]
                assert np.array_equal(codes, e4m3_nearest(x * (np.float32(448.0) / amax))), \
                    "batched fp8 row codes"
                assert np.all(np.isfinite(table[codes]))
    for pool in (kq, vq):
        codes = pool[:, :, : bs * D].reshape(NB, H, bs, D)
        assert np.all(codes.transpose(0, 2, 1, 3)[~written] == 0x7F), "fp8 wrote elsewhere"


def pin_copy_blocks(orc, seed=16):
    rng = np.random.default_rng(seed)
    L, NB, H, bs, D = 3, 10, 2, 16, 64
    ks = [rng.integers(0, 1 << 16, size=(NB, H, bs, D), dtype=np.uint16) for _ in range(L)]
    vs = [rng.integers(0, 1 << 16, size=(NB, H, bs, D), dtype=np.uint16) for _ in range(L)]
    k0 = [k.copy() for k in ks]
    v0 = [v.copy() for v in vs]
    pairs = np.array([[1, 7], [4, 2], [9, 0]], dtype=np.int64)
    orc.copy_blocks(ks, vs, pairs)
    dsts = set(pairs[:, 1].tolist())
    for l in range(L):
        for src, dst in pairs:
            assert np.array_equal(ks[l][dst], k0[l][src]), "K dst != src"
            assert np.array_equal(vs[l][dst], v0[l][src]), "V dst != src"
        for b in range(NB):
            if b not in dsts:
                assert np.array_equal(ks[l][b], k0[l][b]), "K block changed"
                assert np.array_equal(vs[l][b], v0[l][b]), "V block changed"


def pin_swap_blocks(orc, seed=17):
    """Swapping blocks out to a second pool and back restores every byte;
    each destination block equals its source; nothing else changes."""
    rng = np.random.default_rng(seed)
    L, H, bs, D = 2, 2, 8, 64
    gk = [rng.integers(0, 1 << 16, size=(12, H, bs, D), dtype=np.uint16) for _ in range(L)]
    gv = [rng.integers(0, 1 << 16, size=(12, H, bs, D), dtype=np.uint16) for _ in range(L)]
    hk = [rng.integers(0, 1 << 16, size=(5, H, bs, D), dtype=np.uint16) for _ in range(L)]
    hv = [rng.integers(0, 1 << 16, size=(5, H, bs, D), dtype=np.uint16) for _ in range(L)]
    g0 = [x.copy() for x in gk + gv]
    h0 = [x.copy() for x in hk + hv]
    out_map = np.array([[3, 0], [11, 4], [6, 2]], dtype=np.int64)
    orc.swap_blocks(gk, gv, hk, hv, out_map)
    for l in range(L):
        for a, b in out_map:
            assert np.array_equal(hk[l][b], gk[l][a]) and np.array_equal(hv[l][b], gv[l][a])
        for b in (1, 3):
            assert np.array_equal(hk[l][b], h0[l][b]) and np.array_equal(hv[l][b], h0[L + l][b])
    # Clobber the source blocks, swap back in: the original bytes return.
    for l in range(L):
        for a, _ in out_map:
            gk[l][a] = 0
            gv[l][a] = 0
    orc.swap_blocks(hk, hv, gk, gv, out_map[:, ::-1])
    for l in range(L):
        assert np.array_equal(gk[l], g0[l]) and np.array_equal(gv[l], g0[L + l])


def e4m3_table():
    """Value of every e4m3 code, from torch's own float8_e4m3fn conversion."""
    import torch
    return torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()


def e4m3_nearest(x):
    """Brute force: the finite e4m3 code nearest to each float x, ties to the
    even code (the even mantissa), magnitudes above 448 clamped to 448."""
    vals = e4m3_table()
    finite = [c for c in range(256) if np.isfinite(vals[c])]
    fv = vals[finite]
    out = []
    for v in np.asarray(x, dtype=np.float64).reshape(-1):
        v = float(np.clip(v, -448.0, 448.0))
        d = np.abs(fv - v)
        best = np.nonzero(d == d.min())[0]
        cands = [finite[i] for i in best]
        if len(cands) > 1:
            same_sign = [c for c in cands if (c >> 7) == (1 if np.signbit(v) else 0)]
            cands = same_sign or cands
            even = [c for c in cands if c % 2 == 0]
            cands = even or cands
        out.append(cands[0])
    return np.array(out, dtype=np.uint8)


def pin_fp8(orc, seed=18):
    """e4m3 decoding equals torch's for all 256 codes; encoding is the
    brute-force nearest value; a paged fp8 cache written row by row decodes
    like dense attention over the dequantised rows."""
    table = e4m3_table()
    for c in range(256):
        got = orc.e4m3_decode(c)
        assert (np.isnan(got) and np.isnan(table[c])) or got == table[c], f"code {c:#x}"
    rng = np.random.default_rng(seed)
    fv = table[np.isfinite(table)]
    mids = (np.sort(fv)[1:] + np.sort(fv)[:-1]) / 2          # exact ties
    xs = np.concatenate([rng.standard_normal(300) * 10.0 ** rng.uniform(-4, 3, 300),
                         mids[::7], [448.0, 447.99, 464.0, 464.01, 1e4, 2.0 ** -10, 1e-9,
                                     -0.0, 0.0, 2.0 ** -9 * 7.5]]).astype(np.float32)
    got = np.array([orc.e4m3_encode(x) for x in xs], dtype=np.uint8)
    want = e4m3_nearest(xs)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, f"encode differs at {xs[bad[:3]]}: {got[bad[:3]]} vs {want[bad[:3]]}"
    # Paged fp8 cache, written through slots one token at a time.
    H, D, bs = 2, 64, 16
    ctxs = [1, 17, 40]
    nb = sum(-(-c // bs) for c in ctxs) + 2
    tb = bs * D + 4 * bs
    perm = rng.permutation(nb)
    kc = np.full((nb, H, tb), 0x7F, dtype=np.uint8)
    vc = kc.copy()
    bt = np.full((3, 3), -1, dtype=np.int32)
    K, V, nxt = [], [], 0
    for s, c in enumerate(ctxs):
        blocks = perm[nxt: nxt + -(-c // bs)]
        nxt += len(blocks)
        bt[s, : len(blocks)] = blocks
        k = to_storage_bits(rng.standard_normal((c, H, D), dtype=np.float32), "f16")
        v = to_storage_bits(rng.standard_normal((c, H, D), dtype=np.float32), "f16")
        for t in range(c):
            slot = np.array([blocks[t // bs] * bs + t % bs], dtype=np.int64)
            orc.write_kv_fp8(k[t:t + 1], v[t:t + 1], slot, kc, vc, bs)
        K.append(k)
        V.append(v)
    q = to_storage_bits(rng.standard_normal((3, H, D), dtype=np.float32), "f16")
    got = orc.decode_fp8(q, kc, vc, bt, np.array(ctxs, dtype=np.int32), np.float32(0.125), bs)
    for s, c in enumerate(ctxs):
        kd = np.zeros((c, H, D))
        vd = np.zeros((c, H, D))
        for t in range(c):
            b, o = bt[s][t // bs], t % bs
            for h in range(H):
                for pool, raw, dq in ((kc, K[s], kd), (vc, V[s], vd)):
                    codes = pool[b, h, o * D:(o + 1) * D]
                    sc = pool[b, h, bs * D + 4 * o: bs * D + 4 * o + 4].view(np.float32)[0]
                    x = raw[t, h].view(np.float16).astype(np.float32)
                    amax = np.float32(np.max(np.abs(x)))
                    assert sc == amax / np.float32(448.0), "row scale"
                    inv = np.float32(448.0) / amax
                    assert np.array_equal(codes, e4m3_nearest(x * inv)), "row codes"
                    dq[t, h] = table[codes] * np.float64(sc)
                    err = np.abs(dq[t, h] - x)
                    assert np.all(err <= np.abs(x) / 16 + np.float64(sc) * 2.0 ** -9 + 1e-7)
        qf = q[s].view(np.float16).astype(np.float64)
        scores = 0.125 * np.einsum("hd,nhd->hn", qf, kd)
        p = scipy.special.softmax(scores, axis=-1)
        ref = np.einsum("hn,nhd->hd", p, vd)
        assert np.max(np.abs(got[s] - ref)) <= 1e-12, "fp8 decode vs dense"


def pin_grouped_heads(orc, seed=19):
    """Grouped heads: query head h attends to K/V head h // G, as dense
    attention on the unpaged copy with the K/V heads repeated G times."""
    rng = np.random.default_rng(seed)
    for Hk, G, dtype in [(2, 4, "f16"), (1, 3, "f16"), (2, 2, "bf16")]:
        c = paged_case(rng, [1, 20, 75], Hk, 64, 16, dtype=dtype)
        q = to_storage_bits(rng.standard_normal((3, Hk * G, 64), dtype=np.float32), dtype)
        got = orc.decode(q, c["kpool"], c["vpool"], c["bt"], c["ctx"], c["scale"], dtype)
        for s in range(3):
            K = np.repeat(c["K"][s], G, axis=1)
            V = np.repeat(c["V"][s], G, axis=1)
            ref = dense_attention(q[s], K, V, c["scale"], dtype)
            assert np.max(np.abs(got[s] - ref)) <= 1e-12, "grouped heads vs dense"


def pin_grouped_heads_fp8(orc, seed=20):
    """Grouped heads on an fp8 cache: the decode equals the decode of the
    same cache with each K/V head's tiles repeated G times (one K/V head per
    query head), whose fp8 path pin_fp8 ties to dense attention."""
    rng = np.random.default_rng(seed)
    for Hk, G, D, bs in [(2, 3, 64, 16), (1, 4, 128, 8)]:
        ctxs = [1, 20, 47]
        nb = sum(-(-c // bs) for c in ctxs) + 2
        tb = bs * D + 4 * bs
        kc = np.full((nb, Hk, tb), 0x7F, dtype=np.uint8)
        vc = kc.copy()
        bt = np.full((3, max(-(-c // bs) for c in ctxs)), -1, dtype=np.int32)
        perm, nxt = rng.permutation(nb), 0
        for s, c in enumerate(ctxs):
            blocks = perm[nxt: nxt + -(-c // bs)]
            nxt += len(blocks)
            bt[s, : len(blocks)] = blocks
            k = to_storage_bits(rng.standard_normal((c, Hk, D), dtype=np.float32), "f16")
            v = to_storage_bits(rng.standard_normal((c, Hk, D), dtype=np.float32), "f16")
            slots = np.array([blocks[t // bs] * bs + t % bs for t in range(c)], dtype=np.int64)
            orc.write_kv_fp8(k, v, slots, kc, vc, bs)
        q = to_storage_bits(rng.standard_normal((3, Hk * G, D), dtype=np.float32), "f16")
        ctx = np.array(ctxs, dtype=np.int32)
        got = orc.decode_fp8(q, kc, vc, bt, ctx, np.float32(0.1), bs)
        ref = orc.decode_fp8(q, np.repeat(kc, G, axis=1), np.repeat(vc, G, axis=1), bt, ctx,
                             np.float32(0.1), bs)
        assert np.max(np.abs(got - ref)) <= 1e-12, "fp8 grouped heads vs repeated heads"


ALL_PINS = [pin_grouped_heads, pin_grouped_heads_fp8, pin_dense, pin_bruteforce, pin_closed_forms,
            pin_permutation, pin_write_kv, pin_write_kv_batched, pin_copy_blocks,
            pin_swap_blocks, pin_fp8]
