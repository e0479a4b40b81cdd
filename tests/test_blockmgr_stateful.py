"""The native block manager under random serving traces (CPU, hypothesis).

Requests arrive with prompts drawn from a few shared system prompts (prefix
caching) or without token ids, are forked for parallel sampling, append one
or several tokens per step in batches, and finish.  After every operation the
manager must satisfy the pages' rules ("PagedAttention", "The idea: page the
KV cache" and "Sharing and copy-on-write"):
  - a block's reference count is the number of table entries naming it, and
    the free list holds exactly the blocks nobody names;
  - a sequence of L tokens holds ceil(L / block_size) blocks (waste below one
    block);
  - shared blocks are full, except a partial last block shared by forks that
    have not written into it yet;
  - a step's copies target blocks that were free, at most one per sequence;
  - the prefix cache names only held, full blocks;
and the batch calls must agree with the capacity query."""
import numpy as np
from hypothesis import HealthCheck, settings
from hypothesis import strategies as st
from hypothesis.stateful import RuleBasedStateMachine, initialize, invariant, precondition, rule

NUM_BLOCKS, BS = 48, 4
PROMPTS = [[int(x) for x in np.random.default_rng(s).integers(0, 1000, 40)] for s in range(3)]


class ServingTrace(RuleBasedStateMachine):
    @initialize()
    def start(self):
        import paged_kv_cache_343_b200 as pa
        self.pa = pa
        self.bm = pa.BlockManager(NUM_BLOCKS, BS)
        self.live = []
        self.next_id = 0
        self.prompt_of = {}   # seq -> the prompt token ids it was added with (new tokens follow them)

    def _new_id(self):
        self.next_id += 1
        return self.next_id - 1

    @rule(which=st.integers(0, 2), cut=st.integers(1, 40))
    def add_with_prefix(self, which, cut):
        toks = PROMPTS[which][:cut]
        s = self._new_id()
        free = self.bm.num_free()
        try:
            cached = self.bm.add_sequence_with_prefix(s, toks)
        except self.pa.PagedAttnError as e:
            assert e.name == "PA_ERR_OUT_OF_BLOCKS"
            assert self.bm.num_free() == free
            return
        assert cached % BS == 0 and cached <= (len(toks) // BS) * BS
        # the cached prefix is a prefix some held sequence added with the same tokens
        if cached:
            assert any(self.prompt_of.get(o, [])[:cached] == toks[:cached] for o in self.live)
        self.live.append(s)
        self.prompt_of[s] = toks

    @rule(n=st.integers(0, 30))
    def add_plain(self, n):
        s = self._new_id()
        try:
            self.bm.add_sequence(s, n)
        except self.pa.PagedAttnError as e:
            assert e.name == "PA_ERR_OUT_OF_BLOCKS"
            return
        self.live.append(s)

    @precondition(lambda self: self.live)
    @rule(i=st.integers(0, 1000))
    def fork(self, i):
        parent = self.live[i % len(self.live)]
        child = self._new_id()
        self.bm.fork(parent, child)
        self.live.append(child)
        if parent in self.prompt_of:
            self.prompt_of[child] = self.prompt_of[parent]

    @precondition(lambda self: self.live)
    @rule(data=st.data())
    def step(self, data):
        k = data.draw(st.integers(1, len(self.live)))
        batch = data.draw(st.permutations(self.live))[:k]
        several = data.draw(st.booleans())
        counts = [data.draw(st.integers(0, 6)) for _ in batch] if several else None
        need = self.bm.blocks_needed(batch, counts)
        free = self.bm.num_free()
        before = {s: self.bm.block_table(s) for s in self.live}
        lens = {s: self.bm.seq_len(s) for s in batch}
        try:
            if several:
                slots, q_start, pairs = self.bm.append_tokens(batch, counts)
            else:
                slots, pairs = self.bm.append_slots(batch)
                q_start = None
        except self.pa.PagedAttnError as e:
            assert e.name == "PA_ERR_OUT_OF_BLOCKS" and need > free
            assert {s: self.bm.block_table(s) for s in self.live} == before
            return
        assert need <= free and free - self.bm.num_free() == need
        n_new = counts if several else [1] * len(batch)
        assert slots.numel() == sum(n_new)
        if q_start is not None:
            assert q_start.tolist() == [0] + list(np.cumsum(n_new))
        dsts = [int(d) for _, d in pairs.tolist()]
        assert len(set(dsts)) == len(dsts) <= len(batch)
        held_before = {b for t in before.values() for b in t}
        assert not held_before.intersection(dsts)   # copies go to blocks that were free
        for s, c in zip(batch, n_new):
            assert self.bm.seq_len(s) == lens[s] + c
        # every new token's slot lies in its sequence's table at its position
        row = 0
        for s, c in zip(batch, n_new):
            t = self.bm.block_table(s)
            for j in range(c):
                pos = lens[s] + j
                assert int(slots[row]) == t[pos // BS] * BS + pos % BS
                row += 1

    @precondition(lambda self: self.live)
    @rule(i=st.integers(0, 1000))
    def finish(self, i):
        s = self.live.pop(i % len(self.live))
        self.bm.free_sequence(s)
        self.prompt_of.pop(s, None)

    @invariant()
    def pages_rules(self):
        if not hasattr(self, "bm"):
            return
        names = np.zeros(NUM_BLOCKS, np.int64)
        fills = {}
        for s in self.live:
            t = self.bm.block_table(s)
            L = self.bm.seq_len(s)
            assert len(t) == -(-L // BS)
            for i, b in enumerate(t):
                names[b] += 1
                fills.setdefault(b, []).append(min(BS, L - i * BS))
        for b, f in fills.items():  # a shared block is full, or equally filled by all
            assert len(f) == 1 or all(x == BS for x in f) or len(set(f)) == 1
        assert [self.bm.refcount(b) for b in range(NUM_BLOCKS)] == names.tolist()
        assert self.bm.num_free() == int(np.sum(names == 0))
        st_ = self.bm.stats()
        assert st_["held_blocks"] == int(np.sum(names > 0))
        assert st_["max_waste_per_seq"] < BS
        # the cache names only held full blocks: at most one entry per held
        # block that some sequence holds full
        assert st_["cached_blocks"] <= sum(1 for b, f in fills.items() if max(f) == BS)


TestServingTrace = ServingTrace.TestCase
TestServingTrace.settings = settings(max_examples=60, stateful_step_count=40, deadline=None,
                                     suppress_health_check=[HealthCheck.too_slow])
