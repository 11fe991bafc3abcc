"""The host block manager (include/block_manager.h), on the CPU.

The manager's outputs are checked by simulation, not against a second
implementation: a pool of slots holds, for every position written, a value
that stands for that position's key/value row -- a function of the whole
token prefix up to it, as a real K/V row is.  The test applies exactly what a
serving loop would (write the rows of the positions the manager did not take
from the prefix cache, run the copy-on-write copies, write each appended row
at its slot) and checks after every operation that:
  * reading each live sequence's positions through its block table gives the
    values of its own token history (sharing, forks, copy-on-write and prefix
    hits never expose another sequence's rows);
  * every block's reference count equals the number of tables holding it,
    and the free count equals the number of blocks with count 0;
  * a table covers exactly ceil(len / block_size) blocks, and the blocks a
    step writes are held by that sequence alone.
Failed calls (out of blocks, unknown ids) must leave everything unchanged.
"""

import random

import pytest

import paged_kv_cache_473_b200 as pa
from paged_kv_cache_473_b200 import _binding as bnd


def kv_value(tokens):
    """Stand-in for the K/V row of the last position of ``tokens`` (depends on the whole prefix)."""
    return hash(tuple(tokens))


class Sim:
    def __init__(self, num_blocks, bs, seed):
        self.m = pa.BlockManager(num_blocks, bs)
        self.nb, self.bs = num_blocks, bs
        self.pool = {}  # slot -> value
        self.hist = {}  # seq id -> token list
        self.rng = random.Random(seed)
        self.next_id = 0

    # ---- operations ---------------------------------------------------------------
    def add(self, tokens):
        sid = self.next_id
        self.next_id += 1
        before = self.snapshot()
        try:
            cached = self.m.add_sequence(sid, len(tokens), tokens)
        except pa.PagedAttnError as e:
            assert e.status == bnd.PA_ERR_WORKSPACE
            assert self.snapshot() == before
            return None
        assert cached % self.bs == 0 and cached <= len(tokens)
        slots = self.m.slots(sid, 0, len(tokens)).tolist()
        for t in range(cached):  # prefix-cache hits: the rows must already be there
            assert self.pool.get(slots[t]) == kv_value(tokens[: t + 1])
        for t in range(cached, len(tokens)):
            self.pool[slots[t]] = kv_value(tokens[: t + 1])
        self.hist[sid] = list(tokens)
        return sid

    def append(self, sids, with_tokens=True):
        toks = [self.rng.randrange(50) for _ in sids]
        before = self.snapshot()
        try:
            slots, cow = self.m.append_slots(sids, toks if with_tokens else None)
        except pa.PagedAttnError as e:
            assert e.status == bnd.PA_ERR_WORKSPACE
            assert self.snapshot() == before
            return False
        for src, dst in cow.tolist():  # copy-on-write first, as pa_copy_blocks would
            for r in range(self.bs):
                if src * self.bs + r in self.pool:
                    self.pool[dst * self.bs + r] = self.pool[src * self.bs + r]
        assert len(set(slots.tolist())) == len(sids)
        for sid, s, tok in zip(sids, slots.tolist(), toks):
            self.hist[sid].append(tok)
            assert self.m.ref_count(s // self.bs) == 1, "a step writes a block another sequence holds"
            self.pool[s] = kv_value(self.hist[sid])
        return True

    def fork(self, parent):
        child = self.next_id
        self.next_id += 1
        self.m.fork(parent, child)
        self.hist[child] = list(self.hist[parent])
        return child

    def free(self, sid):
        self.m.free(sid)
        del self.hist[sid]

    # ---- checks -------------------------------------------------------------------
    def snapshot(self):
        ids = sorted(self.hist)
        tables = self.m.block_tables(ids, self.max_blocks())[0].tolist() if ids else []
        return (self.m.num_free, tuple(self.m.ref_count(b) for b in range(self.nb)),
                tuple(map(tuple, tables)), tuple(self.m.length(i) for i in ids))

    def max_blocks(self):
        return max(1, max((len(h) + self.bs - 1) // self.bs for h in self.hist.values()) if self.hist else 1)

    def check(self):
        ids = sorted(self.hist)
        refs = [0] * self.nb
        if ids:
            tables, lens = self.m.block_tables(ids, self.max_blocks())
            for i, sid in enumerate(ids):
                h = self.hist[sid]
                assert int(lens[i]) == len(h) == self.m.length(sid)
                row = [int(x) for x in tables[i] if int(x) >= 0]
                assert len(row) == (len(h) + self.bs - 1) // self.bs
                assert len(set(row)) == len(row)
                for b in row:
                    refs[b] += 1
                for t in range(len(h)):
                    slot = row[t // self.bs] * self.bs + t % self.bs
                    assert self.pool.get(slot) == kv_value(h[: t + 1]), f"seq {sid} position {t}"
        assert [self.m.ref_count(b) for b in range(self.nb)] == refs
        assert self.m.num_free == sum(1 for r in refs if r == 0)


@pytest.mark.parametrize("seed", range(12))
@pytest.mark.parametrize("bs", [1, 4, 16])
def test_random_serving_trace(seed, bs):
    """Prompts with shared prefixes, decode steps, forks (parallel sampling),
    frees (completion / preemption) and pool exhaustion, in random order."""
    sim = Sim(num_blocks=40 if bs > 1 else 300, bs=bs, seed=seed)
    rng = sim.rng
    prefixes = [[rng.randrange(50) for _ in range(rng.randrange(1, 3 * bs + 2))] for _ in range(3)]
    for _ in range(250):
        op = rng.random()
        live = sorted(sim.hist)
        if op < 0.25 or not live:
            p = rng.choice(prefixes) if rng.random() < 0.6 else []
            tail = [rng.randrange(50) for _ in range(rng.randrange(0, 2 * bs + 3))]
            if p or tail:
                sim.add(p + tail)
        elif op < 0.65:
            k = rng.randrange(1, min(6, len(live)) + 1)
            sim.append(rng.sample(live, k), with_tokens=rng.random() < 0.8)
        elif op < 0.78:
            sim.fork(rng.choice(live))
        else:
            sim.free(rng.choice(live))
        sim.check()
    for sid in list(sim.hist):
        sim.free(sid)
    sim.check()
    assert sim.m.num_free == sim.nb


def test_fork_then_append_copies_the_shared_partial_block():
    m = pa.BlockManager(8, 4)
    assert m.add_sequence(1, 6) == 0
    tables, _ = m.block_tables([1], 2)
    b0, b1 = tables[0].tolist()
    m.fork(1, 2)
    assert m.ref_count(b0) == 2 and m.ref_count(b1) == 2
    slots, cow = m.append_slots([1])
    assert cow.shape == (1, 2) and int(cow[0, 0]) == b1
    new = int(cow[0, 1])
    assert int(slots[0]) == new * 4 + 2
    assert m.ref_count(b1) == 1 and m.ref_count(new) == 1 and m.ref_count(b0) == 2
    slots, cow = m.append_slots([2])  # the other holder now owns b1 alone: no copy
    assert cow.shape == (0, 2) and int(slots[0]) == b1 * 4 + 2


def test_prefix_cache_hits_only_exact_full_block_prefixes():
    m = pa.BlockManager(16, 4)
    assert m.add_sequence(1, 10, list(range(10))) == 0
    assert m.add_sequence(2, 9, list(range(8)) + [99]) == 8  # two full blocks shared
    assert m.add_sequence(3, 9, [0, 1, 2, 5] + list(range(4, 9))) == 0  # first block differs
    assert m.add_sequence(4, 3, [0, 1, 2]) == 0  # no full block
    t, _ = m.block_tables([1, 2], 3)
    assert t[0, :2].tolist() == t[1, :2].tolist() and t[0, 2] != t[1, 2]
    # A freed prefix stays cached until its blocks are handed out again.
    m.free(1)
    m.free(2)
    assert m.add_sequence(5, 8, list(range(8))) == 8


def test_blocks_filled_by_decode_become_cacheable():
    m = pa.BlockManager(16, 4)
    m.add_sequence(1, 2, [7, 8])
    for tok in [9, 10, 11, 12]:
        m.append_slots([1], [tok])
    assert m.add_sequence(2, 5, [7, 8, 9, 10, 11]) == 4


def test_out_of_blocks_and_bad_ids_change_nothing():
    m = pa.BlockManager(3, 4)
    m.add_sequence(1, 8)
    with pytest.raises(pa.PagedAttnError) as e:
        m.add_sequence(2, 8)
    assert e.value.status == bnd.PA_ERR_WORKSPACE
    assert m.num_free == 1 and m.length(2) == -1
    with pytest.raises(pa.PagedAttnError):
        m.add_sequence(1, 2)  # duplicate id
    m.add_sequence(3, 4)
    with pytest.raises(pa.PagedAttnError) as e:
        m.append_slots([1, 3])  # both need a new block, none free
    assert e.value.status == bnd.PA_ERR_WORKSPACE
    assert m.length(1) == 8 and m.length(3) == 4
    with pytest.raises(pa.PagedAttnError):
        m.append_slots([1, 1])  # repeated id
    with pytest.raises(pa.PagedAttnError):
        m.block_tables([1], 1)  # table too narrow
    with pytest.raises(pa.PagedAttnError):
        m.slots(1, 5, 4)  # past the end
    with pytest.raises(pa.PagedAttnError):
        m.fork(7, 8)
    with pytest.raises(pa.PagedAttnError):
        m.free(42)
    assert pa.BlockManager(1, 1).num_free == 1
    with pytest.raises(pa.PagedAttnError):
        pa.BlockManager(0, 16)


def test_tables_and_slots_feed_the_decode_layout():
    """block_tables/slots give exactly the int32 table rows and int64 slots the
    decode calls take (row-major, -1 padded)."""
    m = pa.BlockManager(10, 16)
    m.add_sequence(5, 20)
    m.add_sequence(9, 1)
    tables, lens = m.block_tables([9, 5], 4)
    assert tables.dtype.is_floating_point is False and tables.shape == (2, 4)
    assert lens.tolist() == [1, 20]
    assert (tables[0, 1:] == -1).all() and (tables[1, 2:] == -1).all()
    s = m.slots(5, 0, 20)
    assert s.tolist() == [int(tables[1, t // 16]) * 16 + t % 16 for t in range(20)]
