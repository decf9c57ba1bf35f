"""A CPU model of the attention kernel's synchronisation (fk_attention.cu):
the load warp's TMA loads and buffer-free waits, the MMA warp's schedule of
MMA issues, commits and mbarrier waits, the two softmax warpgroups, an
in-order tensor-core queue and TMA loads that land in any order, all
interleaved at random.

The mbarrier is modelled by its phase count; a parity wait succeeds when
the current phase's parity differs from the one asked for, as on the GPU.
Every wait that succeeds must have seen the phase it meant (not one two
phases on, which the parity cannot tell apart), every MMA must find its
operands in place (the K/V tile it wants in shared memory, P_j in the S
region, O holding blocks 0..j-1), and no schedule may stall.  Every tile
count a grid can hand a CTA (one or two query tiles, causal or not, up to
eight key blocks) is run under many random interleavings.

The model follows the kernel's load and MMA loops step by step; a change
there must be made here too.  A variant that frees K_j too early (after
tile 0's S_j, whatever tile reads K_j last) is shown to overwrite a tile
an MMA still needs, so the model can catch that class of mistake.
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
    """kfree_after_last=False plants a mistake: K_j is reported free once
    tile 0's S_j is issued, whatever tile reads K_j last."""

    def __init__(self, nkv, rng, kfree_after_last=True):
        self.nkv = nkv
        self.rng = rng
        self.kfree_after_last = kfree_after_last
        names = ("q", "k0", "k1", "v0", "v1", "kfree0", "kfree1", "vfree0", "vfree1", "s0", "s1", "o0", "o1",
                 "p0", "p1", "drain")
        self.bars = {n: Bar(1) for n in names}
        self.tensor = []  # in issue order: ("mma", op) or ("commit", bar)
        self.tma = []     # (buffer, tile)
        self.smem = {}
        self.tmem = {}
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
        """The load warp: Q, then K_j and V_j into buffer j % 2 once the
        MMAs that read K_j-2 / V_j-2 are done."""
        nmax = max(self.nkv)
        self.tma.append(("q", ("q", 0)))
        for j in range(nmax):
            if j >= 2:
                yield from self.wait(f"kfree{j & 1}", (j - 2) >> 1)
            self.tma.append((f"k{j & 1}", ("k", j)))
            if j >= 2:
                yield from self.wait(f"vfree{j & 1}", (j - 2) >> 1)
            self.tma.append((f"v{j & 1}", ("v", j)))

    def mma(self):
        """The MMA warp."""
        nkv = self.nkv
        nmax = max(nkv)
        ntiles = 2 if nkv[1] > 0 else 1
        seen = {"k": 0, "v": 0}

        def last(j):  # the tile that reads K_j and V_j last
            return 1 if j < nkv[1] else 0

        def wait_tile(kind, j):
            if j < seen[kind]:
                return
            yield from self.wait(f"{kind}{j & 1}", j >> 1)
            seen[kind] = j + 1

        def issue_s(i, j):
            self.tensor.append(("mma", ("S", i, j, f"k{j & 1}", ("k", j))))
            self.tensor.append(("commit", f"s{i}"))
            if i == (last(j) if self.kfree_after_last else 0):
                self.tensor.append(("commit", f"kfree{j & 1}"))

        yield from self.wait("q", 0)
        yield from wait_tile("k", 0)
        for i in range(ntiles):
            issue_s(i, 0)
        for j in range(nmax):
            for i in range(2):
                if j < nkv[i]:
                    # the tiles first (long since loaded), then the softmax
                    yield from wait_tile("v", j)
                    if j + 1 < nkv[i]:
                        yield from wait_tile("k", j + 1)
                    yield from self.wait(f"p{i}", j)
                    self.tensor.append(("mma", ("O", i, j, f"v{j & 1}", ("v", j))))
                    if i == last(j):
                        self.tensor.append(("commit", f"vfree{j & 1}"))
                    if j + 1 < nkv[i]:
                        issue_s(i, j + 1)
                    else:
                        self.tensor.append(("commit", f"o{i}"))
        self.tensor.append(("commit", "drain"))
        yield from self.wait("drain", 0)

    def softmax(self, i):
        for j in range(self.nkv[i]):
            yield from self.wait(f"s{i}", j)
            if self.tmem.get(f"S{i}") != ("S", j):
                self.errors.append(f"softmax {i} block {j} found {self.tmem.get(f'S{i}')}")
            for _ in range(self.rng.randint(0, 3)):
                yield "work"
            self.tmem[f"S{i}"] = ("P", j)  # P_i,j over the S columns
            self.bars[f"p{i}"].arrive()
        if self.nkv[i] > 0:
            yield from self.wait(f"o{i}", 0)
            if self.tmem.get(f"O{i}") != self.nkv[i] - 1:
                self.errors.append(f"epilogue {i} found O through block {self.tmem.get(f'O{i}')}")

    def step_tensor(self):
        if not self.tensor:
            return False
        kind, x = self.tensor.pop(0)
        if kind == "commit":
            self.bars[x].arrive()
            return True
        typ, i, j, buf, want = x
        if self.smem.get(buf) != want:
            self.errors.append(f"{typ}{i},{j} read {buf} = {self.smem.get(buf)}, wanted {want}")
        if typ == "O":
            if self.tmem.get(f"S{i}") != ("P", j):
                self.errors.append(f"O{i},{j} read {self.tmem.get(f'S{i}')} as P")
            if self.tmem.get(f"O{i}", -1) != j - 1:
                self.errors.append(f"O{i},{j} accumulated onto block {self.tmem.get(f'O{i}', -1)}")
            self.tmem[f"O{i}"] = j
        else:
            self.tmem[f"S{i}"] = ("S", j)
        return True

    def step_tma(self):
        if not self.tma:
            return False
        buf, _ = self.tma[self.rng.randrange(len(self.tma))]
        first = next(n for n, (b, _) in enumerate(self.tma) if b == buf)  # one buffer's loads land in order
        buf, tile = self.tma.pop(first)
        for kind, x in self.tensor:
            if kind == "mma" and x[3] == buf and x[4] != tile:
                self.errors.append(f"load {tile} over {buf} still wanted by {x[:3]}")
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


def cta_tile_counts(max_blocks=8):
    """(key blocks of query tile 0, of query tile 1) for every CTA of every
    grid the kernel launches with t = 128 .. 128 max_blocks."""
    out = set()
    for nq in range(1, max_blocks + 1):
        for causal in (False, True):
            for pair in range((nq + 1) // 2):
                nkv = tuple(((2 * pair + i + 1) if causal else nq) if 2 * pair + i < nq else 0 for i in range(2))
                out.add(nkv)
    return sorted(out)


@pytest.mark.parametrize("nkv", cta_tile_counts())
def test_schedule_is_race_and_stall_free(nkv):
    for seed in range(150):
        errors = Model(nkv, random.Random(seed)).run()
        assert not errors, (seed, errors[:3])


def test_model_catches_an_early_kfree():
    """With K_j reported free after tile 0's S_j, the load of K_j+2 can
    land while S_1,j still waits in the tensor queue for K_j."""
    found = False
    for seed in range(200):
        if Model((4, 4), random.Random(seed), kfree_after_last=False).run():
            found = True
            break
    assert found
