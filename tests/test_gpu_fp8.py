"""fp8 (e4m3, one fp32 scale per row) KV cache: the CUDA path against the
oracle. Quantised writes and block copies are compared byte for byte (codes
and scale bytes); decode outputs within 2e-3 of the oracle's attention over
the dequantised cache."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_417_b200 as pk
import workloads as wl
from tests.gpu_harness import TOL, max_err, run_step, run_step_fused, to_bits

pytestmark = pytest.mark.gpu

CASES = [
    ("tiny", lambda: wl.tiny(dtype="fp8")),
    ("llama_reduced", lambda: wl.llama_layer(num_seqs=12, num_blocks=1024, dtype="fp8")),
    ("long_reduced", lambda: wl.long_context(num_seqs=3, ctx_range=(3000, 6000),
                                             num_blocks=1500, dtype="fp8")),
    ("prefix_cow", lambda: wl.prefix_cow(num_seqs=16, dtype="fp8")),
    ("full_bs8", lambda: wl.full_step(block_size=8, num_seqs=24, num_layers=2, dtype="fp8")),
    ("full_bs16", lambda: wl.full_step(block_size=16, num_seqs=24, num_layers=2, dtype="fp8")),
    ("full_bs32", lambda: wl.full_step(block_size=32, num_seqs=24, num_layers=2, dtype="fp8")),
    ("d64_bs8", lambda: wl.llama_layer(num_seqs=6, num_blocks=1200, head_dim=64, num_heads=8,
                                       block_size=8, dtype="fp8")),
]


@pytest.mark.parametrize("name,make", CASES, ids=[c[0] for c in CASES])
@pytest.mark.parametrize("fused", [False, True], ids=["separate", "fused"])
@pytest.mark.parametrize("partition", [0, 64])
def test_fp8_matches_oracle(name, make, fused, partition):
    st = make()
    run = run_step_fused if fused else run_step
    outs, d, err = run(st, partition_size=partition)
    assert err == 0
    for li in range(st.num_layers):
        ref, kref, vref = oracle.run_step(st, li)
        assert max_err(outs[li], ref) <= TOL
        assert np.array_equal(to_bits(d["key_caches"][li]), kref)
        assert np.array_equal(to_bits(d["value_caches"][li]), vref)


def test_fp8_full_size_sampled():
    st = wl.llama_layer(dtype="fp8")
    outs, d, err = run_step_fused(st)
    assert err == 0
    ids = sorted({int(np.argmin(st.context_lens)), int(np.argmax(st.context_lens)), 5, 60})
    ref, _, _ = oracle.run_step(wl.subset(st, ids), 0)
    assert max_err(outs[0][torch.as_tensor(ids, device="cuda")], ref) <= TOL


@pytest.mark.parametrize("D", [64, 128])
def test_fp8_write_bf16_rows(D):
    """bf16 rows quantised into an fp8 cache equal the oracle's codes and
    scales byte for byte, including zero rows and large magnitudes."""
    rng = np.random.default_rng(D)
    T, H, bs, NB = 9, 3, 16, 8
    x = rng.standard_normal((2, T, H, D)).astype(np.float32) * 10.0 ** rng.uniform(-3, 3, (2, T, H, 1))
    x[0, 2] = 0.0
    bits = wl.to_storage_bits(x, "bf16")
    slots = rng.permutation(NB * bs)[:T].astype(np.int64)
    slots[4] = -1
    tb = bs * D + 4 * bs
    host_k = np.zeros((NB, H, tb), dtype=np.uint8)
    host_v = np.zeros((NB, H, tb), dtype=np.uint8)
    oracle.write_kv_fp8(bits[0], bits[1], slots, host_k, host_v, bs, io_dtype="bf16")
    kc = pk.Fp8Cache(torch.zeros(NB, H, tb, dtype=torch.uint8, device="cuda"), bs, D,
                     torch.bfloat16)
    vc = pk.Fp8Cache(torch.zeros(NB, H, tb, dtype=torch.uint8, device="cuda"), bs, D,
                     torch.bfloat16)
    dev = [torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).cuda() for b in bits]
    pk.write_kv(dev[0], dev[1], torch.from_numpy(slots).cuda(), kc, vc)
    torch.cuda.synchronize()
    assert np.array_equal(to_bits(kc), host_k) and np.array_equal(to_bits(vc), host_v)


def test_fp8_copy_and_swap_move_scales():
    st = wl.tiny(dtype="fp8")
    outs, d, _ = run_step(st)
    kc, vc = d["key_caches"][0], d["value_caches"][0]
    before = to_bits(kc).copy()
    used = int(st.block_tables[3, 0])
    free = sorted(set(range(st.num_blocks)) - set(st.block_tables.reshape(-1).tolist()))[:2]
    pk.copy_blocks([kc], [vc], torch.tensor([[used, free[0]]], dtype=torch.int64).cuda())
    host = pk.Fp8Cache(torch.zeros(2, *kc.shape[1:], dtype=torch.uint8).pin_memory(),
                       st.block_size, st.head_dim)
    hostv = pk.Fp8Cache(torch.zeros(2, *kc.shape[1:], dtype=torch.uint8).pin_memory(),
                        st.block_size, st.head_dim)
    pk.swap_blocks([kc], [vc], [host], [hostv], torch.tensor([[used, 1]], dtype=torch.int64).cuda())
    torch.cuda.synchronize()
    after = to_bits(kc)
    assert np.array_equal(after[free[0]], before[used])
    assert np.array_equal(to_bits(host)[1], before[used])
