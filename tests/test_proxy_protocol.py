"""A CPU model of the proxy-pass kernel's barrier protocol (proxy_pass.cu), run over random work
shares and completion delays.

The persistent kernel walks a contiguous run of (head pair, 16-block chunk) items. Its roles: the
TMA producer (the last 128 queries of each pair's heads whenever the pair changes, and the key
blocks through a 3-slot ring), the MMA issuer (S_t = Q_t K^T into one of two TMEM buffers per
tile), the softmax warps of each tile (one agent per tile here; the kernel's eight act alike), and
the two K-mean warps that read every key block too. A K slot is released by three parties: the
MMA commit and the two K-mean warps. A pair of an odd GQA group's last head has one tile, so the
second tile's softmax and buffers skip that pair's items. The model replays each role's waits and
arrivals in the kernel's order and checks:
  - every role finishes (no deadlock);
  - no wait finds its barrier two or more phases past the awaited one (parity aliasing);
  - data hazards: an MMA reads the Q tiles of its own pair and the K slot of its own block, and
    neither is reloaded under it; the K-mean warps read the K slot of their block; the softmax reads
    the S buffer of its own block, and a buffer is rewritten only after the softmax freed it.
"""
import random

import pytest

from tests.protocol_sim import Bar, Sim

NS = 3        # K ring depth
CHUNK = 16    # key blocks per item


def items_for(G, h_kv, nb, P, c):
    """The (pair, ntiles, nblk) items CTA c of P runs: the (pair, chunk) list in pair order, each
    CTA a contiguous share."""
    ppg = (G + 1) // 2
    n_chunks = -(-nb // CHUNK)
    I = h_kv * ppg * n_chunks
    lo, hi = c * I // P, (c + 1) * I // P
    out = []
    for it in range(lo, hi):
        pair, chunk = divmod(it, n_chunks)
        pig = pair % ppg
        out.append((pair, 2 if 2 * pig + 1 < G else 1, min(CHUNK, nb - CHUNK * chunk)))
    return out


class ProxyModel(Sim):
    def __init__(self, items, seed, broken=None):
        super().__init__(seed)
        self.items, self.broken = items, broken
        self.q_full, self.q_empty = Bar("q_full", 1), Bar("q_empty", 1)
        self.k_full = [Bar(f"k_full{i}", 1) for i in range(NS)]
        self.k_empty = [Bar(f"k_empty{i}", 3) for i in range(NS)]  # MMA commit + two K-mean warps
        self.s_full = [[Bar(f"s_full{t}{b}", 1) for b in range(2)] for t in range(2)]
        self.s_free = [[Bar(f"s_free{t}{b}", 1) for b in range(2)] for t in range(2)]
        self.mma_done = Bar("mma_done", 1)
        self.qslot = None             # pair whose Q tiles sit in shared memory
        self.kslot = [None] * NS      # key block (running count) a slot holds
        self.s_tag = [[None, None], [None, None]]   # tile block index whose S a buffer holds
        self.s_freed = [[0, 0], [0, 0]]             # uses of each buffer the softmax has freed
        self.tail = 0

    def mma(self, check, on_done):
        check()
        self.tail = max(self.time, self.tail) + self.rng.randint(1, 12)
        self.events.append((self.tail, on_done))

    def commit(self, bar):
        self.tail = max(self.time, self.tail) + 1
        self.events.append((self.tail, bar.arrive))

    def producer(self):
        kc = qn = 0
        prev = None
        for pair, ntiles, nblk in self.items:
            if pair != prev:
                if qn > 0 and self.broken != "no_q_empty_wait":
                    yield (self.q_empty, qn - 1)
                self.qslot = None

                def land_q(pair=pair):
                    self.qslot = pair
                    self.q_full.arrive()
                self.later(self.rng.randint(1, 40), land_q)
                qn += 1
                prev = pair
            for _ in range(nblk):
                st = kc % NS
                if kc >= NS:
                    yield (self.k_empty[st], kc // NS - 1)
                self.kslot[st] = None

                def land_k(st=st, kc=kc):
                    self.kslot[st] = kc
                    self.k_full[st].arrive()
                self.later(self.rng.randint(1, 40), land_k)
                kc += 1
        if qn > 0:
            yield (self.q_full, qn - 1)
        for j in range(max(0, kc - NS), kc):  # never leave with copies in flight
            yield (self.k_full[j % NS], j // NS)

    def issuer(self):
        kc = qn = 0
        tb = [0, 0]
        prev = None
        for pair, ntiles, nblk in self.items:
            if pair != prev:
                if qn > 0:
                    self.commit(self.q_empty)  # the old Q tiles are free once their MMAs finish
                yield (self.q_full, qn)
                qn += 1
                prev = pair
            for _ in range(nblk):
                st = kc % NS
                yield (self.k_full[st], kc // NS)
                for t in range(ntiles):
                    b = tb[t] & 1
                    if tb[t] >= 2:
                        yield (self.s_free[t][b], tb[t] // 2 - 1)

                    def check(pair=pair, st=st, kc=kc):
                        assert self.qslot == pair, ("MMA reads another pair's Q", pair, self.qslot)
                        assert self.kslot[st] == kc, ("MMA reads the wrong K", kc, self.kslot)

                    def done(t=t, b=b, blk=tb[t], chk=check):
                        chk()
                        assert self.s_freed[t][b] >= blk // 2, ("S buffer rewritten before freed", t, b, blk)
                        self.s_tag[t][b] = blk
                    self.mma(check, done)
                    self.commit(self.s_full[t][b])
                    tb[t] += 1
                self.commit(self.k_empty[st])
                kc += 1
        self.commit(self.mma_done)
        yield (self.mma_done, 0)

    def softmax(self, t):
        tb = 0
        for pair, ntiles, nblk in self.items:
            if t >= ntiles:
                continue
            for _ in range(nblk):
                b = tb & 1
                yield (self.s_full[t][b], tb // 2)
                assert self.s_tag[t][b] == tb, ("softmax reads the wrong S", t, tb, self.s_tag[t][b])
                yield None  # the exponentials
                self.s_freed[t][b] += 1
                self.s_free[t][b].arrive()
                tb += 1

    def kmean(self, w):
        kc = 0
        for pair, ntiles, nblk in self.items:
            for _ in range(nblk):
                st = kc % NS
                yield (self.k_full[st], kc // NS)
                assert self.kslot[st] == kc, ("K mean reads the wrong K", w, kc, self.kslot)
                yield None  # the column sums
                assert self.kslot[st] == kc, ("K reloaded under the K mean", w, kc)
                if not (self.broken == "kmean_no_release" and w == 1):
                    self.k_empty[st].arrive()
                kc += 1

    def roles(self):
        return {"producer": self.producer(), "issuer": self.issuer(), "softmax0": self.softmax(0),
                "softmax1": self.softmax(1), "kmean0": self.kmean(0), "kmean1": self.kmean(1)}


@pytest.mark.parametrize("G", [1, 2, 3, 4, 7])
def test_proxy_protocol_random_shares(G):
    rng = random.Random(G)
    for trial in range(120):
        h_kv = rng.randint(1, 3)
        nb = rng.randint(1, 40)
        P = rng.randint(1, 9)
        c = rng.randrange(P)
        items = items_for(G, h_kv, nb, P, c)
        if not items:
            continue
        ProxyModel(items, trial).run()


def test_items_follow_the_contiguous_split():
    # Qwen-like group (7 heads per kv-head): pairs of two heads and a last pair of one
    all_items = [it for c in range(5) for it in items_for(7, 2, 40, 5, c)]
    assert len(all_items) == 2 * 4 * 3
    assert [it[1] for it in all_items[:12]] == [2] * 9 + [1] * 3
    assert sum(it[2] for it in all_items) == 2 * 4 * 40


def test_model_catches_q_reloaded_under_the_mma():
    """Pins of the model: reloading Q without waiting for the MMAs on the old tiles is caught."""
    items = items_for(4, 2, 3, 1, 0)  # four pairs of one short chunk each
    caught = 0
    for seed in range(40):
        try:
            ProxyModel(items, seed, broken="no_q_empty_wait").run()
        except AssertionError as e:
            assert "Q" in str(e) or "phase" in str(e), e
            caught += 1
    assert caught > 0


def test_model_catches_a_missing_k_release():
    with pytest.raises(AssertionError, match="deadlock"):
        ProxyModel(items_for(4, 1, 20, 1, 0), 0, broken="kmean_no_release").run()
