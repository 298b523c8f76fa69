"""The barrier protocol of the tensor-core attention kernel, checked on the CPU.

`attn_tc_kernel` runs one persistent CTA per SM: a TMA producer, one MMA-issuing
warp per query tile and one softmax warpgroup per tile, synchronised only by
mbarriers. This test runs a discrete model of those roles (each a generator that
yields while it waits) under random interleavings, with the mbarrier semantics of
the hardware: a barrier completes a phase after its expected number of arrivals,
and a wait on parity p returns once the phase with that parity has completed.

What is modelled, per tile t (NT tiles) and a ring of STAGES key-block stages:
  producer   per item: the query tile of every tile with rows (after q_empty of
             its previous use), then the item's key blocks in order (after
             kv_empty of the stage's previous use);
  issuer t   per block j: S_t(j) (after kv_full and s_free of block j - 1), then
             P V of block j - 1 (after p_full; at an item's first block after
             o_empty of the previous item); after its own blocks, the item's
             remaining blocks are released once they have landed;
  softmax t  per block: read S (s_full), free it (s_free), write P after the
             previous P V (p_free), signal p_full; at the item's end, read O
             after the last P V and free it (o_empty).
Each shared buffer records who wrote and read it, so an overwrite before use
fails an assertion; a state where no role can move is a deadlock.

The turns at the exponentials (head_dim 64, two tiles) add a pairwise handshake
between the softmax warpgroups that this model leaves out.
"""
import random

import pytest


class Barrier:
    """An mbarrier: `count` arrivals complete a phase."""

    def __init__(self, count):
        self.count, self.arrivals, self.phases = count, 0, 0

    def arrive(self):
        self.arrivals += 1
        if self.arrivals == self.count:
            self.arrivals, self.phases = 0, self.phases + 1

    def passed(self, parity):  # the phase with this parity has completed
        return (self.phases & 1) != parity


class Deadlock(Exception):
    pass


def simulate(items, stages, nt, rng, release_before_last_pv=False, skip_s_free=False):
    """Run the roles over `items` (per item, the key blocks of each tile) until
    all finish. Two planted mistakes for the negative controls:
    `release_before_last_pv` (the issuers release the blocks a tile has no rows
    for before its last P V) and `skip_s_free` (the issuers write S without
    waiting for the softmax to have read the previous S)."""
    bar = {}
    for t in range(nt):
        for name in ("q_full", "q_empty", "s_full", "s_free", "p_full", "p_free", "o_empty"):
            bar[name, t] = Barrier(1)  # the 128 arrivals of a warpgroup are modelled as one
    for s in range(stages):
        bar["kv_full", s] = Barrier(1)
        bar["kv_empty", s] = Barrier(nt)  # one release per issuer
    st = {"S_written": [-1] * nt, "S_read": [-1] * nt, "P_written": [-1] * nt, "P_used": [-1] * nt,
          "O_acc_item": [None] * nt, "O_read_item": [None] * nt, "Q_item": [None] * nt,
          "Q_last_S_item": [None] * nt, "stage_block": {}, "stage_free": {}, "releases": {}}

    def producer():
        g, qn = 0, [0] * nt
        for it, nb in enumerate(items):
            for t in range(nt):
                if nb[t] == 0:
                    continue
                if qn[t] >= 1:
                    while not bar["q_empty", t].passed((qn[t] - 1) & 1):
                        yield
                assert st["Q_item"][t] is None or st["Q_last_S_item"][t] == st["Q_item"][t], "Q overwritten"
                st["Q_item"][t] = it
                bar["q_full", t].arrive()
                qn[t] += 1
            for _ in range(max(nb)):
                s = g % stages
                while not bar["kv_empty", s].passed(((g // stages) & 1) ^ 1):
                    yield
                assert st["stage_free"].get(s, True), "K/V stage overwritten"
                st["stage_block"][s], st["stage_free"][s] = g, False
                bar["kv_full", s].arrive()
                g += 1

    def issuer(t):
        g = cb = qn = 0

        def release(s):
            st["releases"][s] = st["releases"].get(s, 0) + 1
            if st["releases"][s] == nt:
                st["releases"][s], st["stage_free"][s] = 0, True
            bar["kv_empty", s].arrive()

        def pv(i, it):
            gi = cb + i
            while not bar["p_full", t].passed(gi & 1):
                yield
            if i == 0 and qn >= 1:
                while not bar["o_empty", t].passed((qn - 1) & 1):
                    yield
                assert st["O_read_item"][t] == st["O_acc_item"][t], "O overwritten before read"
            if i == 0:
                st["O_acc_item"][t] = it
            assert st["P_written"][t] == gi, "P V before P"
            assert st["stage_block"][(g + i) % stages] == g + i, "stage holds another block"
            st["P_used"][t] = gi
            bar["p_free", t].arrive()
            release((g + i) % stages)

        def remaining(nb, nall):
            for j in range(nb, nall):
                s = (g + j) % stages
                while not bar["kv_full", s].passed(((g + j) // stages) & 1):
                    yield
                release(s)

        for it, nb_all in enumerate(items):
            nall, nb = max(nb_all), nb_all[t]
            if nb > 0:
                while not bar["q_full", t].passed(qn & 1):
                    yield
                assert st["Q_item"][t] == it, "S from another item's queries"
            if release_before_last_pv:
                for j in range(nb):
                    yield from s_mma(t, it, nb, j, g, cb)
                    if j >= 1:
                        yield from pv(j - 1, it)
                yield from remaining(nb, nall)
                if nb > 0:
                    yield from pv(nb - 1, it)
            else:  # as the kernel: S(j) then P V(j - 1) for j = 0 .. nb, then the rest
                for j in range(nb + 1):
                    if j < nb:
                        yield from s_mma(t, it, nb, j, g, cb)
                    if j >= 1:
                        yield from pv(j - 1, it)
                yield from remaining(nb, nall)
            g += nall
            if nb > 0:
                cb += nb
                qn += 1

    def s_mma(t, it, nb, j, g, cb):
        s = (g + j) % stages
        while not bar["kv_full", s].passed(((g + j) // stages) & 1):
            yield
        assert st["stage_block"][s] == g + j, "stage holds another block"
        gj = cb + j
        if gj >= 1 and not skip_s_free:
            while not bar["s_free", t].passed((gj - 1) & 1):
                yield
        assert st["S_read"][t] == gj - 1, "S overwritten before read"
        st["S_written"][t] = gj
        if j == nb - 1:
            st["Q_last_S_item"][t] = it
            bar["q_empty", t].arrive()
        bar["s_full", t].arrive()

    def softmax(t):
        cb = 0
        for it, nb_all in enumerate(items):
            nb = nb_all[t]
            if nb == 0:
                continue
            for j in range(nb):
                gj = cb + j
                while not bar["s_full", t].passed(gj & 1):
                    yield
                assert st["S_written"][t] == gj, "S of another block"
                st["S_read"][t] = gj
                bar["s_free", t].arrive()
                if gj >= 1:
                    while not bar["p_free", t].passed((gj - 1) & 1):
                        yield
                    assert st["P_used"][t] == gj - 1, "P overwritten before use"
                st["P_written"][t] = gj
                bar["p_full", t].arrive()
            while not bar["p_free", t].passed((cb + nb - 1) & 1):
                yield
            assert st["O_acc_item"][t] == it
            st["O_read_item"][t] = it
            bar["o_empty", t].arrive()
            cb += nb

    roles = [producer()] + [issuer(t) for t in range(nt)] + [softmax(t) for t in range(nt)]
    alive = [True] * len(roles)
    idle_rounds = 0
    while any(alive):
        order = [k for k in range(len(roles)) if alive[k]]
        rng.shuffle(order)
        for k in order:
            try:
                for _ in range(rng.randint(1, 3)):
                    next(roles[k])
            except StopIteration:
                alive[k] = False
        idle_rounds += 1
        if idle_rounds > 20000:
            raise Deadlock()


def random_items(rng, nt, decoder):
    """Per item, the key blocks of each of its nt tiles: the decoder's tiles read
    the same blocks (trailing tiles may have no rows); the encoder's causal tiles
    read 0-2 more blocks each than the tile before (in any tile order, since a
    tile's row chunk need not be the item's first), and trailing ones may be empty."""
    items = []
    for _ in range(rng.randint(1, 7)):
        used = rng.randint(1, nt)
        if decoder:
            b = rng.randint(0, 6)
            blocks = [b if i < used else 0 for i in range(nt)]
        else:
            b = [rng.randint(1, 4)]
            for _ in range(1, nt):
                b.append(b[-1] + rng.randint(0, 2))
            blocks = [b[i] if i < used else 0 for i in range(nt)]
            rng.shuffle(blocks)
        items.append(tuple(blocks))
    return items


@pytest.mark.parametrize("nt,stages", [(2, 3), (3, 6), (2, 2), (3, 3)])
def test_protocol_has_no_deadlock_or_overwrite(nt, stages):
    """The kernel's shapes (two tiles with 3 stages at head_dim 64, three tiles
    with 6 stages at head_dim 32) and tighter rings, over random decoder and
    causal encoder item sequences."""
    rng = random.Random(1000 * nt + stages)
    for trial in range(1000):
        items = random_items(rng, nt, decoder=trial % 2 == 0)
        simulate(items, stages, nt, rng)


def test_model_catches_a_misordered_issuer():
    """Negative control: releasing the blocks a tile has no rows for before its
    last P V deadlocks once a tile reads more than a ring's worth of blocks
    beyond another (three causal tiles of 1, 2 and 4 blocks, 3 stages): the
    released-early stages wait for a P V that waits for a stage."""
    rng = random.Random(7)
    with pytest.raises(Deadlock):
        simulate([(1, 2, 4)], 3, 3, rng, release_before_last_pv=True)
    simulate([(1, 2, 4)], 3, 3, rng)  # the kernel's order finishes


def test_model_catches_an_overwrite():
    """Negative control: issuers that write the next S without waiting for the
    softmax to have read the last one are caught overwriting S (some random
    interleavings reach it within a few items)."""
    rng = random.Random(11)
    caught = 0
    for _ in range(50):
        try:
            simulate([(4, 4, 4), (3, 5, 6)], 6, 3, rng, skip_s_free=True)
        except AssertionError as e:
            assert "S overwritten" in str(e)
            caught += 1
    assert caught > 0
