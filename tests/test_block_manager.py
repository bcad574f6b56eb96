"""The C++ block manager against the independent Python allocator of
workloads/ (the bookkeeping the pages describe: free list, ref_count,
block tables, fork, copy-on-write), driven in lockstep by random operations."""
import numpy as np
import pytest

import paged_kv_cache_417_b200 as pk
from paged_kv_cache_417_b200.block_manager import BlockManager
import workloads as wl
from workloads import (BlockAllocator, Sequence, allocate_tokens, append_token,
                       check_invariants, free_sequence)


class PyManager:
    """The same operations on the Python allocator."""

    def __init__(self, nb, bs, order):
        self.a = BlockAllocator(nb, bs, order)
        self.seqs = {}

    def blocks_to_append(self, sid):
        s = self.seqs[sid]
        if s.num_tokens % self.a.block_size == 0:
            return 1
        return 1 if self.a.ref_count[s.block_table[-1]] > 1 else 0

    def blocks_to_allocate(self, sid, n):
        s, bs = self.seqs[sid], self.a.block_size
        return -(-(s.num_tokens + n) // bs) - (-(-s.num_tokens // bs))

    def fork(self, parent, child):
        p = self.seqs[parent]
        self.seqs[child] = Sequence(block_table=[self.a.fork(b) for b in p.block_table],
                                    num_tokens=p.num_tokens)


def same_state(py, cc):
    assert cc.num_free == py.a.num_free
    assert np.array_equal(cc.ref_counts(), py.a.ref_count)
    for sid, s in py.seqs.items():
        assert cc.block_table(sid) == s.block_table
        assert cc.num_tokens(sid) == s.num_tokens
    check_invariants(py.a, list(py.seqs.values()))


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("bs", [8, 16, 32])
def test_lockstep_random_operations(seed, bs):
    rng = np.random.default_rng(seed * 100 + bs)
    nb = 96
    order = rng.permutation(nb)
    py, cc = PyManager(nb, bs, order), BlockManager(nb, bs, order)
    next_id = 0
    for step in range(400):
        op = rng.choice(["new", "fork", "append", "free", "decode"], p=[.2, .1, .35, .1, .25])
        live = sorted(py.seqs)
        if op == "new":
            n = int(rng.integers(0, 3 * bs))
            sid = next_id
            next_id += 1
            py.seqs[sid] = Sequence()
            cc.add_sequence(sid)
            need = py.blocks_to_allocate(sid, n)
            if need <= py.a.num_free:
                allocate_tokens(py.a, py.seqs[sid], n)
                cc.allocate_tokens(sid, n)
            else:
                with pytest.raises(pk.PagedKVError):
                    cc.allocate_tokens(sid, n)
        elif op == "fork" and live:
            parent = int(rng.choice(live))
            py.fork(parent, next_id)
            cc.fork(parent, next_id)
            next_id += 1
        elif op == "append" and live:
            sid = int(rng.choice(live))
            if py.blocks_to_append(sid) <= py.a.num_free:
                want = append_token(py.a, py.seqs[sid])
                got = cc.append_token(sid)
                assert got == (want[0], want[1])
            else:
                with pytest.raises(pk.PagedKVError):
                    cc.append_token(sid)
        elif op == "free" and live:
            sid = int(rng.choice(live))
            free_sequence(py.a, py.seqs.pop(sid))
            cc.free_sequence(sid)
        elif op == "decode" and live:
            batch = [int(x) for x in rng.permutation(live)[: int(rng.integers(1, len(live) + 1))]]
            # Python side, one append per sequence in batch order.
            snap_free = py.a.num_free
            need, drops = 0, {}
            for sid in batch:
                s = py.seqs[sid]
                if s.num_tokens % bs == 0:
                    need += 1
                else:
                    last = s.block_table[-1]
                    if py.a.ref_count[last] - drops.get(last, 0) > 1:
                        need += 1
                        drops[last] = drops.get(last, 0) + 1
            mb = max(-(-(py.seqs[sid].num_tokens + 1) // bs) for sid in batch)
            if need > snap_free:
                with pytest.raises(pk.PagedKVError):
                    cc.prepare_decode(batch, mb)
            else:
                res = cc.prepare_decode(batch, mb)
                pairs = []
                for i, sid in enumerate(batch):
                    slot, pair = append_token(py.a, py.seqs[sid])
                    assert res["slot_mapping"][i] == slot
                    if pair:
                        pairs.append(pair)
                    s = py.seqs[sid]
                    assert res["context_lens"][i] == s.num_tokens
                    row = res["block_tables"][i]
                    assert row[: len(s.block_table)].tolist() == s.block_table
                    assert np.all(row[len(s.block_table):] == -1)
                assert [tuple(p) for p in res["copy_pairs"].tolist()] == pairs
        same_state(py, cc)


def test_errors_leave_state_unchanged():
    cc = BlockManager(4, 16)
    cc.add_sequence(1)
    with pytest.raises(pk.PagedKVError):
        cc.add_sequence(1)
    with pytest.raises(pk.PagedKVError):
        cc.allocate_tokens(1, 5 * 16)          # needs 5 blocks of 4
    assert cc.num_free == 4 and cc.num_tokens(1) == 0
    cc.allocate_tokens(1, 20)                  # 2 blocks, last one partly filled
    cc.fork(1, 2)
    with pytest.raises(pk.PagedKVError):
        cc.allocate_tokens(2, 1)               # would write into a shared block
    with pytest.raises(pk.PagedKVError):
        cc.prepare_decode([1, 1], 4)           # one sequence twice in a step
    with pytest.raises(pk.PagedKVError):
        cc.prepare_decode([1], 1)              # table does not fit
    with pytest.raises(pk.PagedKVError):
        cc.free_sequence(7)
    assert cc.num_free == 2 and cc.ref_count(cc.block_table(1)[0]) == 2
    res = cc.prepare_decode([2, 1], 4)         # 2 copies its shared tail; 1 then owns it
    assert res["copy_pairs"].shape == (1, 2)
    assert res["slot_mapping"][1] == cc.block_table(1)[1] * 16 + 4
    with pytest.raises(ValueError):
        BlockManager(3, 16, free_order=[0, 0, 1])


def test_prefix_sharing_reading_of_the_workload():
    """The prefix workload's reading, through the C++ manager: 8 sequences
    fork one 64-token prefix; each gets a private suffix and a forked
    sibling; one decode step copies exactly the partly filled tails."""
    bs, rng = 16, np.random.default_rng(3)
    cc = BlockManager(256, bs, rng.permutation(256))
    cc.add_sequence(0)
    cc.allocate_tokens(0, 64)
    for s in range(1, 8):
        cc.fork(0, s)
    prefix = cc.block_table(0)
    suffix = rng.integers(1, 40, size=8)
    for s in range(8):
        cc.allocate_tokens(s, int(suffix[s]))
        cc.fork(s, 100 + s)                    # sibling: shares every block
    res = cc.prepare_decode(list(range(8)), 8)
    assert len(res["copy_pairs"]) == int(np.sum(suffix % bs != 0))
    assert not set(res["copy_pairs"][:, 0].tolist()) & set(prefix)
    assert all(cc.ref_count(b) == 16 for b in prefix)   # 8 sequences + 8 siblings


NATIVE_CASES = [
    ("tiny", lambda: wl.tiny()),
    ("llama7b_layer", lambda: wl.llama_layer()),
    ("long_context", lambda: wl.long_context()),
    ("prefix_cow", lambda: wl.prefix_cow()),
    ("full_step_bs8", lambda: wl.full_step(block_size=8, num_layers=1)),
    ("full_step_bs16", lambda: wl.full_step(block_size=16, num_layers=1)),
    ("full_step_bs32", lambda: wl.full_step(block_size=32, num_layers=1)),
]


@pytest.mark.parametrize("name,make", NATIVE_CASES, ids=[c[0] for c in NATIVE_CASES])
def test_native_step_inputs_equal_python_allocator(name, make):
    """The benchmark's default inputs: the C++ block manager, replaying each
    workload's allocation history, produces the same block tables, context
    lengths, slots and copy-on-write pairs as the Python allocator. Where the
    workload forks a sibling for each partly filled last block, the C++
    sibling holds the whole pre-step sequence (the Python one its last block
    only): reference counts differ by exactly those extra holdings."""
    import bench
    st = make()
    got = bench.native_inputs(st)
    for k in bench.INTEGER_INPUTS:
        assert np.array_equal(got[k], getattr(st, k)), k
    extra = np.zeros(st.num_blocks, dtype=np.int64)
    if st.meta["fork_partial_tail"]:
        bs = st.block_size
        pre = st.context_lens.astype(np.int64) - 1
        for s in range(st.num_seqs):
            if pre[s] % bs:
                n_pre = -(-pre[s] // bs)
                table = st.block_tables[s, :n_pre].copy()
                if st.copy_pairs.shape[0]:
                    moved = dict(st.copy_pairs.tolist())
                    inv = {dst: src for src, dst in moved.items()}
                    table[-1] = inv.get(int(table[-1]), table[-1])
                extra[table[:-1]] += 1
    assert np.array_equal(got["ref_count"], st.ref_count + extra)
