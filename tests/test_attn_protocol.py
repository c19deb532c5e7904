"""A CPU model of the block-sparse attention kernel's barrier protocol (sparse_attn.cu), run over
random tile masks and random completion delays.

The kernel's roles (the K producer with its 2-slot ring, the V producer with its 3-slot ring, one
MMA issuer per tile, the softmax warps of each tile with their exp2 turns) talk only through
mbarriers, and a wait tests a phase's parity, not its number. This model replays each role's
waits and arrivals in the kernel's order, as one agent per role (the four softmax warps of a
tile act alike), with TMA fills and tcgen05 MMAs completing after random delays (one issuer's
MMAs complete in issue order). It checks:
  - every role finishes (no deadlock) for any mix of steps that one tile, the other or both take;
  - a waiter never finds its barrier two or more phases past the one it waits for (a parity
    test would then mistake an older completion for the awaited one);
  - data hazards: a QK^T reads the K slot filled for its own step and a PV the V slot of its
    step, and neither slot is refilled under the MMA; the softmax reads S of its own block; a
    QK^T overwrites S_t (and the P packed into it) only after the softmax has read that S and
    the PV has consumed that P.
A change to the kernel's waits or releases belongs here first: the model of an earlier, dropped
design failed these checks (a tile skipping steps let a ring run two uses ahead) before that
design ran on a GPU.
"""
import random

import pytest

from tests.protocol_sim import Bar, Sim

NSK, NSV = 2, 3


class Model(Sim):
    def __init__(self, masks, ntiles, seed, broken=None):
        super().__init__(seed)
        self.broken = broken  # a deliberate protocol mistake, for the tests that pin the model
        self.masks, self.ntiles = masks, ntiles
        self.q_full = Bar("q_full", 1)
        self.k_full = [Bar(f"k_full{i}", 1) for i in range(NSK)]
        self.k_empty = [Bar(f"k_empty{i}", ntiles) for i in range(NSK)]
        self.v_full = [Bar(f"v_full{i}", 1) for i in range(NSV)]
        self.v_empty = [Bar(f"v_empty{i}", ntiles) for i in range(NSV)]
        self.s_full = [Bar(f"s_full{t}", 1) for t in range(2)]
        self.p_full = [Bar(f"p_full{t}", 1) for t in range(2)]
        self.o_done = [Bar(f"o_done{t}", 1) for t in range(2)]
        self.turn = [Bar(f"turn{t}", 1) for t in range(2)]
        self.kslot = [None] * NSK  # step whose K the slot holds (None while a fill is in flight)
        self.vslot = [None] * NSV
        self.s_tag = [None, None]  # block (per-tile index) whose S sits in S_t
        self.p_tag = [None, None]  # block whose P sits in S_t
        self.s_reads = [0, 0]  # blocks whose S the softmax has read
        self.pv_done = [0, 0]  # PVs completed
        self.tail = [0, 0]  # completion time of each issuer's last MMA

    # ---------------------------------------------------------------- asynchronous units
    def fill(self, slots, full, st, step):
        slots[st] = None

        def land():
            slots[st] = step
            full[st].arrive()
        self.later(self.rng.randint(1, 40), land)

    def mma(self, t, check_issue, on_done):
        check_issue()
        done = max(self.time, self.tail[t]) + self.rng.randint(1, 12)
        self.tail[t] = done
        self.events.append((done, on_done))

    def commit(self, t, bar):
        done = max(self.time, self.tail[t]) + 1
        self.tail[t] = done
        self.events.append((done, bar.arrive))

    # ---------------------------------------------------------------- roles
    def k_producer(self):
        self.later(self.rng.randint(1, 40), self.q_full.arrive)
        n = len(self.masks)
        for step in range(n):
            st = step % NSK
            if step >= NSK:
                yield (self.k_empty[st], step // NSK - 1)
            self.fill(self.kslot, self.k_full, st, step)
        yield (self.q_full, 0)
        for i in range(max(0, n - NSK), n):  # never leave with copies in flight
            yield (self.k_full[i % NSK], i // NSK)

    def v_producer(self):
        n = len(self.masks)
        for step in range(n):
            st = step % NSV
            if step >= NSV:
                yield (self.v_empty[st], step // NSV - 1)
            self.fill(self.vslot, self.v_full, st, step)
        for i in range(max(0, n - NSV), n):
            yield (self.v_full[i % NSV], i // NSV)

    def issuer(self, t):
        bit = 1 << t
        yield (self.q_full, 0)
        pv_n = qk_n = 0
        prev_mask = 0
        for step in range(len(self.masks) + 1):
            more = step < len(self.masks)
            mask = self.masks[step] if more else 0
            st, prev_vs = step % NSK, (step + NSV - 1) % NSV
            if step > 0:
                use = (prev_mask & bit) != 0
                yield (self.v_full[prev_vs], (step - 1) // NSV)  # V first
                if use:
                    yield (self.p_full[t], pv_n)
                    b, vstep = pv_n, step - 1

                    def chk_pv(b=b, vstep=vstep, vs=prev_vs):
                        assert self.vslot[vs] == vstep, ("PV reads the wrong V", t, vstep, self.vslot)
                        assert self.p_tag[t] == b, ("PV reads the wrong P", t, b, self.p_tag[t])

                    def pv_done(b=b, chk=chk_pv):
                        chk()
                        self.pv_done[t] = b + 1
                    self.mma(t, chk_pv, pv_done)
                    pv_n += 1
                    self.commit(t, self.v_empty[prev_vs])
                else:
                    self.v_empty[prev_vs].arrive()
            if not more:
                break
            yield (self.k_full[st], step // NSK)
            if mask & bit:
                b = qk_n

                def chk_qk(step=step, st=st):
                    assert self.kslot[st] == step, ("QK reads the wrong K", t, step, self.kslot)

                def qk_done(b=b, chk=chk_qk):
                    chk()
                    # S_t (and the P packed into it) is overwritten: the previous block's S must
                    # have been read and its P consumed
                    assert self.s_reads[t] >= b, ("S overwritten before it was read", t, b)
                    assert self.pv_done[t] >= b, ("P overwritten before its PV", t, b)
                    self.s_tag[t] = b
                    self.p_tag[t] = None
                self.mma(t, chk_qk, qk_done)
                qk_n += 1
                self.commit(t, self.s_full[t])
                self.commit(t, self.k_empty[st])
            elif self.broken != ("skip_k_release", t):
                self.k_empty[st].arrive()
            prev_mask = mask
        self.commit(t, self.o_done[t])
        yield (self.o_done[t], 0)

    def softmax(self, t):
        turns = self.ntiles == 2
        i = 0
        for j, m in enumerate(self.masks):
            # tile 0 exponentiates first at each step: it waits for tile 1's hand-off of the
            # step before, tile 1 for tile 0's of this step
            turn_k = j - 1 if t == 0 else j
            if not (m >> t) & 1:
                if turns:
                    if turn_k >= 0:
                        yield (self.turn[t], turn_k)
                    self.turn[t ^ 1].arrive()
                continue
            yield (self.s_full[t], i)
            assert self.s_tag[t] == i, ("softmax reads the wrong S", t, i, self.s_tag[t])
            self.s_reads[t] = i + 1
            if turns and turn_k >= 0:
                yield (self.turn[t], turn_k)
            yield None  # the exponentials
            if turns:
                self.turn[t ^ 1].arrive()
            if self.broken == "p_signalled_before_stored":
                self.p_full[t].arrive()
                yield None
                self.p_tag[t] = i
            else:
                self.p_tag[t] = i
                self.p_full[t].arrive()
            i += 1
        yield (self.o_done[t], 0)

    def roles(self):
        roles = {"kp": self.k_producer(), "vp": self.v_producer()}
        for t in range(self.ntiles):
            roles[f"mma{t}"] = self.issuer(t)
            roles[f"softmax{t}"] = self.softmax(t)
        return roles


def random_masks(rng, L, ntiles):
    if ntiles == 1:
        return [1] * L
    p = rng.random()
    while True:
        masks = []
        for _ in range(L):
            r = rng.random()
            masks.append(3 if r < p else (1 if r < p + (1 - p) / 2 else 2))
        if any(m & 1 for m in masks) and any(m & 2 for m in masks):  # every tile has a block
            return masks


@pytest.mark.parametrize("seed", range(4))
def test_protocol_random_walks(seed):
    rng = random.Random(seed)
    for trial in range(300):
        L = rng.randint(1, 48)
        ntiles = 2 if rng.random() < 0.85 else 1
        if ntiles == 2 and L < 2:
            L = 2
        Model(random_masks(rng, L, ntiles), ntiles, seed * 1000 + trial).run()


@pytest.mark.parametrize("masks", [[3] * 40, [1, 2] * 20, [1] * 20 + [2] * 20, [2, 1, 1, 1, 3, 2, 2, 2, 3]])
def test_protocol_fixed_walks(masks):
    for seed in range(20):
        Model(masks, 2, seed).run()


def test_model_catches_a_lost_release():
    """The model is pinned by planted mistakes: a tile that skips a step without releasing the K
    slot (the plain arrive the kernel makes for a block it skips) stalls the K producer."""
    with pytest.raises(AssertionError, match="deadlock"):
        Model([3, 1, 1, 1, 3], 2, 0, broken=("skip_k_release", 1)).run()


def test_model_catches_p_signalled_before_it_is_stored():
    caught = 0
    for seed in range(40):
        try:
            Model([3] * 6, 2, seed, broken="p_signalled_before_stored").run()
        except AssertionError as e:
            assert "wrong P" in str(e), e
            caught += 1
    assert caught > 0
