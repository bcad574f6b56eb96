"""Pins of the CPU oracle to things other than itself (no GPU needed).

* the pages' worked figures: the K/V sizing arithmetic and the block-table
  sketch ("vLLM基础", §2.3 and §2.5; fixtures in tests/golden/);
* dense attention through scipy's softmax on the unpaged copy;
* brute force in 50-digit decimal arithmetic on tiny inputs;
* closed forms (ctx = 1, scale = 0, equal keys, two tokens, one dominant
  token) and invariance under a permutation of physical block ids;
* numpy's and torch's own fp16 / bf16 widening;
* planted mistakes: mutated copies of the oracle must fail at least one pin.
"""
import json
import os
import subprocess

import numpy as np
import pytest

import oracle
from oracle import Oracle
from tests import paged_cases as pc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
ORACLE_SRC = os.path.join(os.path.dirname(os.path.dirname(__file__)), "oracle", "oracle.c")


@pytest.fixture(scope="module")
def orc():
    return oracle.default()


@pytest.mark.parametrize("pin", pc.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(orc, pin):
    pin(orc)


def test_widen_f16_all_patterns(orc):
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([orc.widen(int(b), "f16") for b in bits])
    both_nan = np.isnan(ref) & np.isnan(got)
    assert np.all(both_nan | (got == ref))
    assert np.array_equal(np.signbit(got[~both_nan]), np.signbit(ref[~both_nan]))


def test_widen_bf16_matches_torch(orc):
    torch = pytest.importorskip("torch")
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    got = np.array([orc.widen(int(b), "bf16") for b in bits])
    both_nan = np.isnan(ref) & np.isnan(got)
    assert np.all(both_nan | (got == ref))


def test_kv_sizing_matches_pages(orc):
    g = json.load(open(os.path.join(GOLDEN, "kv_sizing.json")))
    for c in g["cases"]:
        b = orc.kv_cache_bytes(c["layers"], c["tokens"], c["heads"], c["head_dim"],
                               c["elem_bytes"])
        if c["exact_bytes"] is not None:
            assert b == c["exact_bytes"], c["where"]
        assert round(b / 2 ** 30, c["decimals"]) == c["printed"], c["where"]
    w = g["waste"]
    waste = 100.0 * (1 - w["used_tokens"] / w["allocated_tokens"])
    assert round(waste, w["decimals"]) == w["printed_percent"]


def test_block_table_sketch(orc):
    """The pages' sketch: seq_1 -> physical [3, 7, 12], seq_2 -> [5, 9]."""
    g = json.load(open(os.path.join(GOLDEN, "block_table_sketch.json")))
    bs = g["block_size"]
    t1, t2 = g["tables"]["seq_1"], g["tables"]["seq_2"]
    rng = np.random.default_rng(21)
    H, D, NB = 2, 64, 16
    ctx = [40, 20]
    nan = np.uint16(0x7E00)
    kpool = np.full((NB, H, bs, D), nan, dtype=np.uint16)
    vpool = kpool.copy()
    K, V = [], []
    for tab, n in zip((t1, t2), ctx):
        k = pc.to_storage_bits(rng.standard_normal((n, H, D), dtype=np.float32), "f16")
        v = pc.to_storage_bits(rng.standard_normal((n, H, D), dtype=np.float32), "f16")
        for j in range(n):
            kpool[tab[j // bs], :, j % bs] = k[j]
            vpool[tab[j // bs], :, j % bs] = v[j]
        K.append(k)
        V.append(v)
    bt = np.array([t1, t2 + [-1]], dtype=np.int32)
    q = pc.to_storage_bits(rng.standard_normal((2, H, D), dtype=np.float32), "f16")
    got = orc.decode(q, kpool, vpool, bt, np.array(ctx, dtype=np.int32), np.float32(0.125))
    for s in range(2):
        ref = pc.brute_force(q[s], K[s], V[s], np.float32(0.125))
        assert np.max(np.abs(got[s] - ref)) <= 1e-12
        dense = pc.dense_attention(q[s], K[s], V[s], np.float32(0.125))
        assert np.max(np.abs(got[s] - dense)) <= 1e-12


def test_nan_poison_never_read(orc):
    """Unused blocks and slots past the last token hold NaN; the output is
    finite, so the oracle reads none of them."""
    rng = np.random.default_rng(22)
    c = pc.paged_case(rng, [1, 9, 16, 17, 63], 2, 64, 16, num_blocks=20)
    got = orc.decode(c["q"], c["kpool"], c["vpool"], c["bt"], c["ctx"], c["scale"])
    assert np.all(np.isfinite(got))


def test_empty_context_is_zero(orc):
    rng = np.random.default_rng(23)
    c = pc.paged_case(rng, [0, 5], 2, 64, 16)
    got = orc.decode(c["q"], c["kpool"], c["vpool"], c["bt"], c["ctx"], c["scale"])
    assert np.all(got[0] == 0.0) and np.all(np.isfinite(got[1]))


def test_bad_block_id_is_reported(orc):
    rng = np.random.default_rng(24)
    c = pc.paged_case(rng, [20], 1, 64, 16)
    c["bt"][0, 1] = c["kpool"].shape[0]
    with pytest.raises(ValueError):
        orc.decode(c["q"], c["kpool"], c["vpool"], c["bt"], c["ctx"], c["scale"])


# Planted mistakes: (name, text in oracle.c, replacement).
MUTANTS = [
    ("dropped_scale", "w[j] = scale * dot;", "w[j] = dot;"),
    ("no_max_shift", "w[j] = exp(w[j] - m);", "w[j] = exp(w[j]);"),
    ("softmax_sign", "w[j] = exp(w[j] - m);", "w[j] = exp(m - w[j]);"),
    ("pv_uses_keys", "acc += w[j] * V[(size_t)j * head_dim + d];",
     "acc += w[j] * K[(size_t)j * head_dim + d];"),
    ("qk_uses_values", "dot += q[d] * K[(size_t)j * head_dim + d];",
     "dot += q[d] * V[(size_t)j * head_dim + d];"),
    ("no_normalise", "out[d] = acc / z;", "out[d] = acc;"),
    ("slot_offset", "* block_size + j % block_size) * head_dim);",
     "* block_size + (j + 1) % block_size) * head_dim);"),
    ("head_index", "(((block * num_kv_heads + kvh) * block_size + j % block_size)",
     "(((block * num_kv_heads + 0) * block_size + j % block_size)"),
    ("table_index", "int64_t block = table[j / block_size];",
     "int64_t block = table[(j / block_size + 1) % table_len];"),
    ("fp8_table_index", "int64_t block = table[j / block_size];",
     "int64_t block = table[(j / block_size + 1) % table_len];", 1),
    ("write_offset", "offset = slot % block_size;", "offset = 0;"),
    ("fp8_write_offset", "offset = slot % block_size;", "offset = 0;", 1),
    ("fp8_scale_ignored", "* head_dim + d]) * sk;", "* head_dim + d]);"),
    ("fp8_value_scale_from_key", "* head_dim + d]) * sv;", "* head_dim + d]) * sk;"),
    ("e4m3_ties_up", "double m = rint((a / ldexp(1.0, e) - 1.0) * 8.0);",
     "double m = floor((a / ldexp(1.0, e) - 1.0) * 8.0 + 0.5);"),
    ("e4m3_subnormal_step", "double m = rint(a * 512.0);", "double m = rint(a * 256.0);"),
    ("e4m3_bias", "v = ldexp((double)(8 + m), e - 10);", "v = ldexp((double)(8 + m), e - 11);"),
    ("fp8_row_scale", "*scale = amax / 448.0f;", "*scale = amax / 440.0f;"),
    ("fp8_no_saturation", "if (a >= 448.0)\n        return sign | 0x7e;",
     "if (a >= 480.0)\n        return sign | 0x7e;"),
    ("write_source_row_ignores_token", "size_t src = (size_t)((t * num_heads + h) * head_dim);",
     "size_t src = (size_t)((0 * num_heads + h) * head_dim);", 0),
    ("fp8_write_source_row_ignores_token",
     "size_t src = (size_t)((t * num_heads + h) * head_dim);",
     "size_t src = (size_t)((0 * num_heads + h) * head_dim);", 1),
    ("write_value_from_key", "memcpy(value_cache + dst, value + src,",
     "memcpy(value_cache + dst, key + src,"),
    ("copy_value_from_key", "memcpy(value_caches[l] + dst * block_elems, value_caches[l] + src",
     "memcpy(value_caches[l] + dst * block_elems, key_caches[l] + src"),
    ("swap_value_from_key", "memcpy(dst_v[l] + b * block_elems, src_v[l] + a * block_elems,",
     "memcpy(dst_v[l] + b * block_elems, src_k[l] + a * block_elems,"),
    ("swap_wrong_dst", "memcpy(dst_k[l] + b * block_elems, src_k[l] + a * block_elems,",
     "memcpy(dst_k[l] + a % dst_blocks * block_elems, src_k[l] + a * block_elems,"),
    ("gqa_head_map", "context_lens[s], h / group, scale);",
     "context_lens[s], h % num_kv_heads, scale);", 0),
    ("fp8_gqa_head_map", "context_lens[s], h / group, scale);",
     "context_lens[s], h % num_kv_heads, scale);", 1),
    ("f16_exponent_bias", "v = ldexp((double)(f | 0x400), e - 25);",
     "v = ldexp((double)(f | 0x400), e - 24);"),
]


def _plant(src, old, new, occurrence):
    """Replace the occurrence-th (0-based) copy of `old`; with occurrence
    None, `old` must be unique."""
    if occurrence is None:
        assert src.count(old) == 1, "mutation anchor not unique"
        return src.replace(old, new)
    pos = -1
    for _ in range(occurrence + 1):
        pos = src.index(old, pos + 1)
    return src[:pos] + new + src[pos + len(old):]


@pytest.mark.parametrize("mutant", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(tmp_path, mutant):
    name, old, new = mutant[:3]
    occurrence = mutant[3] if len(mutant) > 3 else None
    src = open(ORACLE_SRC).read()
    if occurrence is None and src.count(old) > 1:
        occurrence = 0
    path = tmp_path / "oracle_mut.c"
    path.write_text(_plant(src, old, new, occurrence))
    lib = tmp_path / "liboracle_mut.so"
    subprocess.run(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11", str(path),
                    "-o", str(lib), "-lm"], check=True)
    mut = Oracle(str(lib))
    caught = []
    for pin in pc.ALL_PINS:
        try:
            pin(mut)
        except (AssertionError, ValueError) as e:
            caught.append((pin.__name__, str(e)[:60]))
    if name == "f16_exponent_bias":
        bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)[::97]
        ref = bits.view(np.float16).astype(np.float64)
        got = np.array([mut.widen(int(b)) for b in bits])
        if not np.all((np.isnan(ref) & np.isnan(got)) | (got == ref)):
            caught.append(("widen", "differs from numpy"))
    assert caught, f"no pin caught the planted mistake {name}"
