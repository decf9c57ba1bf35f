"""A CPU model of the attention kernel's synchronisation (fk_attention.cu):
the load warp's TMA loads and buffer-free waits, the MMA warp's schedule of
MMA issues, commits and mbarrier waits, the two softmax warpgroups and their
epilogues, an in-order tensor-core queue and TMA loads that land in any
order, all interleaved at random.

The blocks are persistent: each one walks a list of units (a pair of query
tiles of one slice), so every barrier's phases run on from one unit to the
next, the K and V buffers are filled by one tile counter across units, Q is
reloaded for each unit once the tensor cores are done with the previous
one's S products, and a unit's first O product overwrites the accumulator
the previous unit's epilogue read.

The mbarrier is modelled by its phase count; a parity wait succeeds when
the current phase's parity differs from the one asked for, as on the GPU.
Every wait that succeeds must have seen the phase it meant (not one two
phases on, which the parity cannot tell apart), every MMA must find its
operands in place (Q and the K/V tile of its unit in shared memory, P_j in
the S region, O holding blocks 0..j-1 of the same unit, or the previous
unit's O already read by its epilogue), and no schedule may stall.  Every
tile count a grid can hand a unit (one or two query tiles, causal or not,
up to eight key blocks) is run alone and in sequences of units, under many
random interleavings.

The model follows the kernel's load and MMA loops step by step; a change
there must be made here too.  Planted mistakes (K_j freed after tile 0's S_j
whatever tile reads K_j last; Q reloaded without waiting for the previous
unit's S products) are shown to be caught.
"""
import random

import pytest


class Bar:
    def __init__(self, count):
        self.count = self.pending = count
        self.phase = 0  # completed phases

    def arrive(self):
        self.pending -= 1
        if self.pending == 0:
            self.phase += 1
            self.pending = self.count

    def ready(self, parity):
        return (self.phase & 1) != parity


class Model:
    """units: (key blocks of query tile 0, of query tile 1) per unit, in the
    order the block walks them.  kfree_after_last=False plants a mistake:
    K_j is reported free once tile 0's S_j is issued, whatever tile reads
    K_j last.  qfree=False plants another: the next unit's Q is loaded
    without waiting for the previous unit's S products."""

    def __init__(self, units, rng, kfree_after_last=True, qfree=True):
        self.units = [tuple(u) for u in units]
        self.rng = rng
        self.kfree_after_last = kfree_after_last
        self.qfree = qfree
        names = ("q", "qfree", "k0", "k1", "v0", "v1", "kfree0", "kfree1", "vfree0", "vfree1", "s0", "s1",
                 "o0", "o1", "p0", "p1", "drain")
        self.bars = {n: Bar(1) for n in names}
        self.tensor = []  # in issue order: ("mma", op) or ("commit", bar)
        self.tma = []     # (buffer, tile)
        self.smem = {}
        self.tmem = {}    # "S<i>": ("S"|"P", unit, j); "O<i>": (unit, j); "Oread<i>": unit
        self.errors = []

    def wait(self, bar, k):
        """Wait for phase k of `bar` by its parity, after a random delay."""
        b = self.bars[bar]
        for _ in range(self.rng.randint(0, 2)):
            yield "delay"
        while not b.ready(k & 1):
            yield "blocked"
        if b.phase != k + 1:
            self.errors.append(f"wait on {bar} for phase {k} passed with {b.phase} phases complete")

    def loader(self):
        """The load warp: per unit, Q once the previous unit's S products
        are done, then K_j and V_j into buffer g % 2 (g counting tiles
        across units) once the MMAs that read tile g-2 are done."""
        g = 0
        for u, nkv in enumerate(self.units):
            if u > 0 and self.qfree:
                yield from self.wait("qfree", u - 1)
            self.tma.append(("q", ("q", u)))
            for j in range(max(nkv)):
                if g >= 2:
                    yield from self.wait(f"kfree{g & 1}", (g - 2) >> 1)
                self.tma.append((f"k{g & 1}", ("k", u, j)))
                if g >= 2:
                    yield from self.wait(f"vfree{g & 1}", (g - 2) >> 1)
                self.tma.append((f"v{g & 1}", ("v", u, j)))
                g += 1

    def mma(self):
        """The MMA warp."""
        seen = {"k": 0, "v": 0}  # tiles (counted across units) seen in shared memory
        cnt = {"s0": 0, "s1": 0, "p0": 0, "p1": 0}
        g0 = 0  # global index of the unit's first K/V tile

        def wait_tile(kind, g):
            if g < seen[kind]:
                return
            yield from self.wait(f"{kind}{g & 1}", g >> 1)
            seen[kind] = g + 1

        for u, nkv in enumerate(self.units):
            ntiles = 2 if nkv[1] > 0 else 1
            s_left = nkv[0] + nkv[1]  # S products of the unit still to issue

            def last(j):  # the tile that reads K_j and V_j last
                return 1 if j < nkv[1] else 0

            def issue_s(i, j):
                nonlocal s_left
                self.tensor.append(("mma", ("S", i, j, u, f"k{(g0 + j) & 1}", ("k", u, j))))
                self.tensor.append(("commit", f"s{i}"))
                if i == (last(j) if self.kfree_after_last else 0):
                    self.tensor.append(("commit", f"kfree{(g0 + j) & 1}"))
                s_left -= 1
                if s_left == 0:
                    self.tensor.append(("commit", "qfree"))

            yield from self.wait("q", u)
            yield from wait_tile("k", g0)
            for i in range(ntiles):
                issue_s(i, 0)
            for j in range(max(nkv)):
                for i in range(2):
                    if j < nkv[i]:
                        yield from wait_tile("v", g0 + j)
                        if j + 1 < nkv[i]:
                            yield from wait_tile("k", g0 + j + 1)
                        yield from self.wait(f"p{i}", cnt[f"p{i}"])
                        cnt[f"p{i}"] += 1
                        self.tensor.append(("mma", ("O", i, j, u, f"v{(g0 + j) & 1}", ("v", u, j))))
                        if i == last(j):
                            self.tensor.append(("commit", f"vfree{(g0 + j) & 1}"))
                        if j + 1 < nkv[i]:
                            issue_s(i, j + 1)
                        else:
                            self.tensor.append(("commit", f"o{i}"))
            g0 += max(nkv)
        self.tensor.append(("commit", "drain"))
        yield from self.wait("drain", 0)

    def softmax(self, i):
        ns = no = 0
        for u, nkv in enumerate(self.units):
            for j in range(nkv[i]):
                yield from self.wait(f"s{i}", ns)
                ns += 1
                if self.tmem.get(f"S{i}") != ("S", u, j):
                    self.errors.append(f"softmax {i} unit {u} block {j} found {self.tmem.get(f'S{i}')}")
                for _ in range(self.rng.randint(0, 3)):
                    yield "work"
                self.tmem[f"S{i}"] = ("P", u, j)  # P_i,j over the S columns
                self.bars[f"p{i}"].arrive()
            if nkv[i] > 0:
                yield from self.wait(f"o{i}", no)
                no += 1
                if self.tmem.get(f"O{i}") != (u, nkv[i] - 1):
                    self.errors.append(f"epilogue {i} of unit {u} found O {self.tmem.get(f'O{i}')}")
                for _ in range(self.rng.randint(0, 3)):
                    yield "work"
                self.tmem[f"Oread{i}"] = u

    def step_tensor(self):
        if not self.tensor:
            return False
        kind, x = self.tensor.pop(0)
        if kind == "commit":
            self.bars[x].arrive()
            return True
        typ, i, j, u, buf, want = x
        if self.smem.get(buf) != want:
            self.errors.append(f"{typ}{i},{j} of unit {u} read {buf} = {self.smem.get(buf)}, wanted {want}")
        if typ == "O":
            if self.tmem.get(f"S{i}") != ("P", u, j):
                self.errors.append(f"O{i},{j} of unit {u} read {self.tmem.get(f'S{i}')} as P")
            if j == 0:
                prev = self.tmem.get(f"O{i}")
                if prev is not None and self.tmem.get(f"Oread{i}") != prev[0]:
                    self.errors.append(f"O{i},0 of unit {u} overwrote unit {prev[0]}'s O before its epilogue")
            elif self.tmem.get(f"O{i}") != (u, j - 1):
                self.errors.append(f"O{i},{j} of unit {u} accumulated onto {self.tmem.get(f'O{i}')}")
            self.tmem[f"O{i}"] = (u, j)
        else:
            if self.smem.get("q") != ("q", u):
                self.errors.append(f"S{i},{j} of unit {u} read Q = {self.smem.get('q')}")
            self.tmem[f"S{i}"] = ("S", u, j)
        return True

    def step_tma(self):
        if not self.tma:
            return False
        buf, _ = self.tma[self.rng.randrange(len(self.tma))]
        first = next(n for n, (b, _) in enumerate(self.tma) if b == buf)  # one buffer's loads land in order
        buf, tile = self.tma.pop(first)
        for kind, x in self.tensor:
            if kind == "mma" and x[4] == buf and x[5] != tile:
                self.errors.append(f"load {tile} over {buf} still wanted by {x[:4]}")
            if kind == "mma" and buf == "q" and x[0] == "S" and tile != ("q", x[3]):
                self.errors.append(f"load {tile} over Q still wanted by {x[:4]}")
        self.smem[buf] = tile
        self.bars[buf].arrive()
        return True

    def run(self):
        live = {"loader": self.loader(), "mma": self.mma(), "softmax0": self.softmax(0),
                "softmax1": self.softmax(1)}
        idle = 0
        while live or self.tensor or self.tma:
            c = self.rng.choice(list(live) + ["tensor", "tma"])
            if c == "tensor":
                moved = self.step_tensor()
            elif c == "tma":
                moved = self.step_tma()
            else:
                try:
                    moved = next(live[c]) != "blocked"
                except StopIteration:
                    del live[c]
                    moved = True
            idle = 0 if moved else idle + 1
            if idle > 1000:
                self.errors.append(f"stalled: {sorted(live)} waiting, tensor queue {self.tensor[:1]}")
                break
        return self.errors


def unit_tile_counts(max_blocks=8):
    """(key blocks of query tile 0, of query tile 1) for every unit of every
    grid the kernel launches with t = 128 .. 128 max_blocks."""
    out = set()
    for nq in range(1, max_blocks + 1):
        for causal in (False, True):
            for pair in range((nq + 1) // 2):
                nkv = tuple(((2 * pair + i + 1) if causal else nq) if 2 * pair + i < nq else 0 for i in range(2))
                out.add(nkv)
    return sorted(out)


@pytest.mark.parametrize("nkv", unit_tile_counts())
def test_schedule_is_race_and_stall_free(nkv):
    for seed in range(150):
        errors = Model([nkv], random.Random(seed)).run()
        assert not errors, (seed, errors[:3])


def test_persistent_sequences_of_units_are_race_and_stall_free():
    """Random sequences of two to five units of every shape, as a persistent
    block walks them (long ones first and short ones after, or any mix)."""
    shapes = unit_tile_counts()
    rng = random.Random(7)
    for trial in range(400):
        units = [rng.choice(shapes) for _ in range(rng.randint(2, 5))]
        errors = Model(units, random.Random(trial)).run()
        assert not errors, (units, trial, errors[:3])


def test_model_catches_an_early_kfree():
    """With K_j reported free after tile 0's S_j, the load of K_j+2 can
    land while S_1,j still waits in the tensor queue for K_j."""
    found = False
    for seed in range(200):
        if Model([(4, 4)], random.Random(seed), kfree_after_last=False).run():
            found = True
            break
    assert found


def test_model_catches_a_q_reload_before_the_s_products_are_done():
    found = False
    for seed in range(300):
        if Model([(3, 3), (2, 2)], random.Random(seed), qfree=False).run():
            found = True
            break
    assert found
