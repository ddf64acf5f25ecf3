"""The chunk kernel's synchronization protocol, as a model on the CPU.

Every role of `chunk_kernel` (the bulk-copy producer, the Q loader, the
decode warps, the MMA thread, the two softmax tiles) is a generator of the
same waits, arrivals, copies, MMAs and commits the kernel issues, in the same
order, with the same barrier indices and parities.  A scheduler runs them in
random interleavings:

* an mbarrier completes a phase when its arrivals (and transaction bytes)
  are in; a parity wait succeeds exactly when the hardware's would, and the
  model fails if that ever differs from "the awaited phase has completed"
  (a wait one or two phases off is the classic hang);
* the tensor pipe may run MMAs out of order except per accumulator, and a
  commit arrives once everything issued before it has run;
* every shared-memory or TMEM buffer carries a version: a read must see the
  version it expects, and a write may not land before every reader of the
  previous version has read it.

Deadlock, a parity alias or a stale read fails the test.  Taking out any one
of the kernel's waits must make some schedule fail (so the model is not
vacuous).
"""

import random

import pytest


class Bar:
    def __init__(self, count):
        self.count, self.pending, self.done, self.tx = count, count, 0, 0

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0
        self._check()

    def _check(self):
        if self.pending == 0 and self.tx == 0:
            self.done += 1
            self.pending = self.count


DECODE_WARPS = 8                               # decode warps of the kernel; each arrives once
ROW_WARPS = 4                                  # softmax warps of one 128-row tile


class Model:
    def __init__(self, blocks, n_tiles, n_units, seed, lag):
        self.rng = random.Random(seed)
        self.blocks, self.NT, self.nu, self.lag = blocks, n_tiles, n_units, lag
        self.B = {}
        for u in range(n_units):
            self.B[("RF", u)] = Bar(1)
            self.B[("RE", u)] = Bar(DECODE_WARPS)
        for i in range(2):
            self.B[("KR", i)] = Bar(DECODE_WARPS)
            self.B[("KF", i)] = Bar(1)
            self.B[("SF", i)] = Bar(1)
            self.B[("PF", i)] = Bar(ROW_WARPS)
            self.B[("PD", i)] = Bar(1)
        for name, n in (("VR", DECODE_WARPS), ("VF", 1), ("QR", 1), ("QF", 1)):
            self.B[name] = Bar(n)
        self.pipe, self.copies, self.buf, self.reads, self.seq = [], [], {}, {}, 0

    def write(self, buf, ver, readers):
        if buf in self.buf:
            missing = readers(self.buf[buf]) - self.reads.get(buf, set())
            assert not missing, f"{buf} v{ver} written before v{self.buf[buf]} was read by {missing}"
        self.buf[buf] = ver
        self.reads[buf] = set()

    def read(self, buf, ver, tag):
        assert self.buf.get(buf) == ver, f"{tag} read {buf} v{self.buf.get(buf)}, wanted v{ver}"
        self.reads.setdefault(buf, set()).add(tag)

    def run(self, roles):
        state = {n: None for n in roles}
        alive = set(roles)
        for _ in range(10 ** 6):
            if not (alive or self.pipe or self.copies):
                return
            choices = []
            for n in alive:
                op = state[n]
                if op is None or op[0] != "wait":
                    choices.append(("role", n))
                    continue
                bar, k = self.B[op[1]], op[2]
                hw, true = (bar.done & 1) != (k & 1), bar.done > k
                assert hw == true, f"parity alias: {n} waits phase {k} of {op[1]}, {bar.done} done"
                if hw:
                    choices.append(("role", n))
            for i, op in enumerate(self.pipe):
                earlier = [o for o in self.pipe if o["seq"] < op["seq"]]
                if op["kind"] == "commit":
                    if not any(o["kind"] != "commit" for o in earlier):
                        choices.append(("pipe", i))
                elif not any(o["kind"] != "commit" and o["acc"] == op["acc"] for o in earlier):
                    choices.append(("pipe", i))
            choices += [("copy", i) for i in range(len(self.copies))]
            assert choices, "deadlock: " + ", ".join(f"{n}: {state[n]}" for n in alive)
            roles_only = [c for c in choices if c[0] == "role"]
            c = (self.rng.choice(roles_only) if roles_only and self.rng.random() < self.lag
                 else self.rng.choice(choices))
            if c[0] == "role":
                n = c[1]
                try:
                    op = next(roles[n])
                except StopIteration:
                    alive.discard(n)
                    continue
                state[n] = op
                if op[0] == "arrive":
                    self.B[op[1]].arrive()
                elif op[0] == "expect_tx":
                    self.B[op[1]].tx += 1
                    self.B[op[1]].arrive()
                elif op[0] == "copy":
                    self.copies.append((self.B[op[1]], op[2]))
                elif op[0] in ("mma", "commit"):
                    self.seq += 1
                    if op[0] == "mma":
                        self.pipe.append(dict(kind="mma", acc=op[1], fn=op[2], seq=self.seq))
                    else:
                        self.pipe.append(dict(kind="commit", fn=self.B[op[1]].arrive, seq=self.seq))
                elif op[0] == "do":
                    op[1]()
            elif c[0] == "pipe":
                self.pipe.pop(c[1])["fn"]()
            else:
                bar, fn = self.copies.pop(c[1])
                fn()
                bar.tx -= 1
                bar._check()
        raise AssertionError("schedule did not finish")


def roles_of(m, drop=None, shift=None):
    """The kernel's roles for the block list m.blocks = [(segment, first, last)],
    one role per warp that waits.  `drop` names one wait to leave out, `shift`
    one wait to aim a phase too late (the mutation checks)."""
    blocks, NT, nu = m.blocks, m.NT, m.nu
    nb = len(blocks)
    seg_of = [b[0] for b in blocks]
    seg_blocks = {}
    for i, b in enumerate(blocks):
        seg_blocks.setdefault(b[0], []).append(i)
    DW, RW = range(DECODE_WARPS), range(ROW_WARPS)
    # ring order: K(0), then K(k + 1), V(k) for each block k
    units = [("K", 0)] if nb else []
    for v in range(nb):
        if v + 1 < nb:
            units.append(("K", v + 1))
        units.append(("V", v))

    def wait(name, bar, k):
        return [] if drop == name else [("wait", bar, k + (shift == name))]

    def producer():
        for n, (typ, blk) in enumerate(units):
            slot = n % nu
            if n >= nu:
                yield from wait("ring_empty", ("RE", slot), n // nu - 1)
            yield ("expect_tx", ("RF", slot))
            yield ("copy", ("RF", slot), lambda slot=slot, typ=typ, blk=blk: m.write(
                ("ring", slot), (typ, blk), lambda p: {("dec", w) for w in DW}))

    def qloader():
        for s in range(len(seg_blocks)):
            if s > 0:
                yield from wait("q_free", "QF", s - 1)
            yield ("expect_tx", "QR")
            yield ("copy", "QR", lambda s=s: m.write(
                "Q", s, lambda p: {("qk", t, i) for i in seg_blocks[p] for t in range(NT)}))

    def decode(w):
        # warp w decodes its 16-token slice of every unit
        kb = vb = 0
        for n, (typ, blk) in enumerate(units):
            slot = n % nu
            yield from wait("ring_full", ("RF", slot), n // nu)
            if typ == "K":
                if kb >= 2:
                    yield from wait("k_free", ("KF", kb & 1), (kb >> 1) - 1)
                yield ("do", lambda slot=slot, blk=blk: (
                    m.read(("ring", slot), ("K", blk), ("dec", w)),
                    m.write(("K", blk & 1, w), blk, lambda p: {("qk", t, p) for t in range(NT)})))
                yield ("arrive", ("KR", kb & 1))
                kb += 1
            else:
                if vb >= 1:
                    yield from wait("v_free", "VF", vb - 1)
                yield ("do", lambda slot=slot, blk=blk: (
                    m.read(("ring", slot), ("V", blk), ("dec", w)),
                    m.write(("V", w), blk, lambda p: {("pv", t, p) for t in range(NT)})))
                yield ("arrive", "VR")
                vb += 1
            yield ("arrive", ("RE", slot))

    def qk(t, k):
        def fn():
            m.read("Q", seg_of[k], ("qk", t, k))
            for w in DW:
                m.read(("K", k & 1, w), k, ("qk", t, k))
            # S overwrites the P of block k - 1, which its softmax and P V read
            m.write(("S", t), k, lambda p: {("pv", t, p)} | {("sm", t, p, w) for w in RW})
        return [("mma", ("S", t), fn), ("commit", ("SF", t))]

    def pv(t, k):
        first = blocks[k][1]

        def fn():
            for w in RW:
                m.read(("P", t, w), k, ("pv", t, k))
            for w in DW:
                m.read(("V", w), k, ("pv", t, k))
            m.reads.setdefault(("S", t), set()).add(("pv", t, k))
            for w in RW:
                o = ("O", t, w)
                if first:
                    prev = m.buf.get(o)
                    assert prev is None or ("epi", t, prev) in m.reads.get(o, set()), "O overwritten unread"
                else:
                    assert m.buf.get(o) == k - 1, f"P V({k}) accumulates onto O v{m.buf.get(o)}"
                m.buf[o] = k
                m.reads[o] = set()
        return [("mma", ("O", t), fn), ("commit", ("PD", t))]

    def mma():
        if not nb:
            return
        yield from wait("q_ready", "QR", 0)
        sq = 1
        yield from wait("k_ready", ("KR", 0), 0)
        for t in range(NT):
            yield from qk(t, 0)
        yield ("commit", ("KF", 0))
        if blocks[0][2]:
            yield ("commit", "QF")
        for k in range(nb):
            nxt = k + 1 < nb
            boundary = nxt and blocks[k + 1][1]
            yield from wait("v_ready", "VR", k)
            yield from wait("p_full", ("PF", 0), k)
            yield from pv(0, k)
            if nxt and not boundary:
                yield from wait("k_ready", ("KR", (k + 1) & 1), (k + 1) >> 1)
                yield from wait("pv_done", ("PD", 0), k)
                yield from qk(0, k + 1)
            if NT == 2:
                yield from wait("p_full", ("PF", 1), k)
                yield from pv(1, k)
            yield ("commit", "VF")
            if nxt:
                if boundary:
                    yield from wait("q_ready", "QR", sq)
                    sq += 1
                    yield from wait("k_ready", ("KR", (k + 1) & 1), (k + 1) >> 1)
                    yield from wait("pv_done", ("PD", 0), k)
                    yield from qk(0, k + 1)
                if NT == 2:
                    yield from wait("pv_done", ("PD", 1), k)
                    yield from qk(1, k + 1)
                yield ("commit", ("KF", (k + 1) & 1))
                if blocks[k + 1][2]:
                    yield ("commit", "QF")

    def softmax(t, w):
        # warp w of tile t owns 32 rows of S, P and O
        for k in range(nb):
            yield from wait("s_full", ("SF", t), k)

            def f(k=k):
                m.read(("S", t), k, ("sm", t, k, w))
                if not blocks[k][1]:                            # a rescale reads and writes O
                    assert m.buf.get(("O", t, w)) == k - 1, "rescale before the previous P V finished"
                m.buf[("P", t, w)] = k
            yield ("do", f)
            yield ("arrive", ("PF", t))
            if blocks[k][2]:
                yield from wait("epilogue_pv", ("PD", t), k)
                yield ("do", lambda k=k: m.read(("O", t, w), k, ("epi", t, k)))

    roles = {"producer": producer(), "q": qloader(), "mma": mma()}
    for w in DW:
        roles[f"decode{w}"] = decode(w)
    for t in range(NT):
        for w in RW:
            roles[f"softmax{t}.{w}"] = softmax(t, w)
    return roles


def block_list(segments):
    return [(s, j == 0, j == n - 1) for s, n in enumerate(segments) for j in range(n)]


SEGMENTS = [[1], [3], [28], [5, 23], [1, 1, 1], [27, 1], [1, 27], [2, 2, 2, 2]]


@pytest.mark.parametrize("segments", SEGMENTS, ids=lambda s: "-".join(map(str, s)))
@pytest.mark.parametrize("n_tiles", [1, 2])
@pytest.mark.parametrize("n_units", [3, 5])
def test_protocol_holds(segments, n_tiles, n_units):
    for seed in range(8):
        m = Model(block_list(segments), n_tiles, n_units, seed, lag=(seed % 4) * 0.3)
        m.run(roles_of(m))


@pytest.mark.parametrize("drop", ["ring_empty", "q_free", "k_free", "v_free", "pv_done", "epilogue_pv",
                                  "p_full", "v_ready", "k_ready", "s_full"])
def test_every_wait_is_needed(drop):
    failed = False
    for segments in ([3], [5, 23], [27, 1]):
        for seed in range(40):
            m = Model(block_list(segments), 2, 3, seed, lag=(seed % 4) * 0.3)
            try:
                m.run(roles_of(m, drop=drop))
            except AssertionError:
                failed = True
                break
        if failed:
            break
    assert failed, f"leaving out the {drop} wait went unnoticed"


@pytest.mark.parametrize("shift", ["ring_empty", "ring_full", "k_free", "v_free", "pv_done", "p_full",
                                   "v_ready", "k_ready", "s_full", "q_ready"])
def test_every_phase_is_right(shift):
    """A wait aimed one phase late either hangs or aliases the parity."""
    with pytest.raises(AssertionError):
        for seed in range(10):
            m = Model(block_list([5, 23]), 2, 3, seed, lag=0.3)
            m.run(roles_of(m, shift=shift))
