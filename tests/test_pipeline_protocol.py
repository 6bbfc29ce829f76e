"""The mbarrier hand-off protocols of the persistent GEMMs, simulated on the CPU.

Each role of a kernel (TMA producer, MMA issuer, decoder warps, epilogue warps) is
written here as a sequence of the waits and arrivals it performs, with the counts,
parities and ring sizes of the kernel source (k_tc_gemm.cu, k_tc_gemm_lowp.cu).  A
scheduler runs the roles in random interleavings under mbarrier semantics (a phase
completes when its pending arrivals and transaction bytes reach zero; a parity wait on
phase parity P passes once the phase in progress has the other parity), and checks:
  * every role finishes (no deadlock);
  * a waiter never sees a barrier that has already run two phases past the one it waits
    for (the parity would then be ambiguous);
  * no producer overwrites a buffer (shared-memory stage, TMEM stage, accumulator) that a
    consumer of its previous contents has not released.
This checks the design of the counts and parities, not the compiled kernels.
"""
import random

import pytest


class Barrier:
    def __init__(self, name, count):
        self.name, self.count = name, count
        self.pending, self.tx, self.completed = count, 0, 0

    def _maybe_complete(self):
        if self.pending == 0 and self.tx == 0:
            self.completed += 1
            self.pending = self.count

    def arrive(self):
        assert self.pending > 0, self.name
        self.pending -= 1
        self._maybe_complete()

    def arrive_expect_tx(self, nbytes):
        self.tx += nbytes
        self.arrive()

    def complete_tx(self, nbytes):
        assert self.tx >= nbytes, self.name
        self.tx -= nbytes
        self._maybe_complete()

    def passes(self, parity, want_phase):
        """try_wait.parity: the phase in progress has parity completed % 2."""
        ok = (self.completed % 2) != parity
        if ok and want_phase is not None:
            assert self.completed <= want_phase + 1, f"{self.name}: ran past phase {want_phase}"
        return ok


class Buffers:
    """Readers still owed per (buffer, slot); a producer may only fill a slot nobody reads."""

    def __init__(self):
        self.readers = {}

    def fill(self, key, n_readers):
        assert self.readers.get(key, 0) == 0, f"{key} overwritten while still being read"
        self.readers[key] = n_readers

    def release(self, key):
        assert self.readers.get(key, 0) > 0, f"{key} released twice"
        self.readers[key] -= 1


def wait(bar, parity, phase):
    """A role step: block until bar passes the parity wait (phase = index of the awaited
    completion, for the overrun check)."""
    return ("wait", bar, parity, phase)


class Async:
    """Work that completes later: TMA loads land in any order; the completions an MMA
    thread's commits report come in issue order (a commit tracks every earlier MMA)."""

    def __init__(self):
        self.loads, self.mma = [], []

    def __bool__(self):
        return bool(self.loads or self.mma)

    def step(self, rng):
        if self.mma and (not self.loads or rng.random() < 0.5):
            self.mma.pop(0)()
        else:
            self.loads.pop(rng.randrange(len(self.loads)))()


def run(roles, q, seed, max_steps=200000, end_check=False):
    """roles: name -> generator of steps; q: the Async the roles hand delayed completions to.
    end_check: when every role has finished (the CTA leaves), no load or MMA completion may
    still be pending (it would land in released shared or tensor memory)."""
    rng = random.Random(seed)
    blocked = {}
    live = dict(roles)
    for _ in range(max_steps):
        if not live and end_check:
            assert not q, f"{len(q.loads)} loads and {len(q.mma)} MMA completions pending after the last role left"
        if not live and not q:
            return
        ready = []
        for name, gen in live.items():
            b = blocked.get(name)
            if b is None or b[1].passes(b[2], b[3]):
                ready.append(name)
        choices = ready + (["<async>"] if q else [])
        assert choices, f"deadlock: blocked {sorted((n, b[1].name) for n, b in blocked.items())}"
        pick = rng.choice(choices)
        if pick == "<async>":
            q.step(rng)
            continue
        blocked.pop(pick, None)
        try:
            step = next(live[pick])
        except StopIteration:
            del live[pick]
            continue
        if step is not None and step[0] == "wait":
            blocked[pick] = step
    raise AssertionError("no progress")


# ---------------------------------------------------------------- the bf16 GEMM (k_tc_gemm.cu)

class Ranges:
    """Byte ranges of a shared-memory ring still being read; a producer may only fill a
    range that overlaps none of them."""

    def __init__(self):
        self.live = []

    def fill(self, off, n):
        for o, m in self.live:
            assert off + n <= o or o + m <= off, f"[{off}, {off + n}) overwrites [{o}, {o + m}) while it is read"
        self.live.append((off, n))

    def release(self, off, n):
        self.live.remove((off, n))


def bf16_gemm(tile_bytes, nkb, cap, slots=16, nbuf=2, bug=None):
    """tile_bytes: the k-block buffer size of each tile (weight boxes + token terms of its
    padded rows); cap: the ring's bytes; slots: barrier pairs (k-blocks in flight at most);
    nbuf: accumulator buffers (one where two do not fit in TMEM: paired weight tiles of
    256 token columns).  The producer allocates each k-block's buffer from the ring (KbRing)
    and waits for the oldest k-blocks until its footprint fits beside theirs (buffers are
    released in allocation order, so that is exactly when it overlaps none of them)."""
    n_tiles = len(tile_bytes)
    full = [Barrier(f"full{s}", 1) for s in range(slots)]
    empty = [Barrier(f"empty{s}", 1) for s in range(slots)]
    acc_full = [Barrier(f"acc_full{b}", 1) for b in range(nbuf)]
    acc_empty = [Barrier(f"acc_empty{b}", 4) for b in range(nbuf)]
    bufs, ranges, q = Buffers(), Ranges(), Async()
    acc_done = {}

    def ring():
        """KbRing::take: (offset, bytes, footprint incl. a skipped tail)."""
        head = 0
        for t in range(n_tiles):
            for _ in range(nkb):
                n = tile_bytes[t]
                if head + n > cap:
                    foot, off, head = cap - head + n, 0, n
                else:
                    foot, off, head = n, head, head + n
                yield off, n, foot

    def producer():
        released, in_use, foot_of = 0, 0, {}
        for it, (off, n, foot) in enumerate(ring()):
            s = it % slots
            in_use += foot
            while released < it and ((in_use > cap and bug != "no_footprint_check") or it - released >= slots):
                yield wait(empty[released % slots], (released // slots) & 1, released // slots)
                in_use -= foot_of[released]
                released += 1
            ranges.fill(off, n)
            foot_of[it] = foot
            full[s].arrive_expect_tx(n)
            q.loads.append(lambda s=s, n=n: full[s].complete_tx(n))

    def mma():
        it = 0
        offs = ((o, n) for o, n, _ in ring())
        for j in range(n_tiles):
            buf = j % nbuf
            yield wait(acc_empty[buf], ((j // nbuf) & 1) ^ 1, j // nbuf - 1)
            bufs.fill(("acc", buf), 4)
            acc_done[buf] = 0
            for kb in range(nkb):
                s = it % slots
                off, n = next(offs)
                yield wait(full[s], (it // slots) & 1, it // slots)

                def done(s=s, buf=buf, off=off, n=n):
                    acc_done[buf] += 1
                    ranges.release(off, n)
                    empty[s].arrive()
                q.mma.append(done)
                it += 1
            q.mma.append(lambda b=buf: acc_full[b].arrive())

    def epilogue(w):
        for j in range(n_tiles):
            buf = j % nbuf
            yield wait(acc_full[buf], (j // nbuf) & 1, j // nbuf)
            assert acc_done[buf] == nkb, "epilogue read an accumulator before its MMAs completed"
            bufs.release(("acc", buf))
            acc_empty[buf].arrive()

    roles = {"tma": producer(), "mma": mma()}
    roles.update({f"epi{w}": epilogue(w) for w in range(4)})
    return roles, q


# ---------------------------------------------------------------- the 8-bit GEMM (k_tc_gemm_lowp.cu)

def lowp_gemm(n_tiles, nkb, stages, t_stages=4, dec_warps=8):
    f_full = [Barrier(f"f_full{s}", 1) for s in range(stages)]
    f_empty = [Barrier(f"f_empty{s}", dec_warps + 1) for s in range(stages)]
    t_full = [Barrier(f"t_full{s}", dec_warps) for s in range(t_stages)]
    t_empty = [Barrier(f"t_empty{s}", 1) for s in range(t_stages)]
    acc_full = [Barrier(f"acc_full{b}", 1) for b in range(2)]
    acc_empty = [Barrier(f"acc_empty{b}", 4) for b in range(2)]
    bufs, q = Buffers(), Async()
    acc_done = {}

    def producer():
        it = 0
        for t in range(n_tiles):
            for kb in range(nkb):
                s = it % stages
                yield wait(f_empty[s], ((it // stages) & 1) ^ 1, it // stages - 1)
                bufs.fill(("smem", s), dec_warps + 1)  # the decoders read the codes, the MMAs the tokens
                f_full[s].arrive_expect_tx(96)
                q.loads.append(lambda s=s: f_full[s].complete_tx(96))
                it += 1

    def mma():
        it = 0
        for j in range(n_tiles):
            buf = j & 1
            yield wait(acc_empty[buf], ((j >> 1) & 1) ^ 1, (j >> 1) - 1)
            bufs.fill(("acc", buf), 4)
            acc_done[buf] = 0
            for kb in range(nkb):
                s, ts = it % stages, it % t_stages
                yield wait(t_full[ts], (it // t_stages) & 1, it // t_stages)
                yield wait(f_full[s], (it // stages) & 1, it // stages)
                assert tmem_writes.get(ts) == (it, dec_warps), "MMA read a TMEM stage not fully written"

                def done(s=s, ts=ts, buf=buf):
                    acc_done[buf] += 1
                    bufs.release(("tmem", ts))
                    t_empty[ts].arrive()
                    bufs.release(("smem", s))
                    f_empty[s].arrive()
                q.mma.append(done)
                it += 1
            q.mma.append(lambda b=buf: acc_full[b].arrive())

    def decoder(w):
        it = 0
        for t in range(n_tiles):
            for kb in range(nkb):
                s, ts = it % stages, it % t_stages
                yield wait(f_full[s], (it // stages) & 1, it // stages)
                yield wait(t_empty[ts], ((it // t_stages) & 1) ^ 1, it // t_stages - 1)
                write_tmem(ts, it)
                bufs.release(("smem", s))
                f_empty[s].arrive()
                t_full[ts].arrive()
                it += 1

    tmem_writes = {}

    def write_tmem(ts, it):
        # each decoder warp writes its part of TMEM stage ts for iteration it; the first
        # write fills the stage (one reader: the MMA), the MMA checks all parts are there
        last, n = tmem_writes.get(ts, (None, 0))
        if last != it:
            bufs.fill(("tmem", ts), 1)
            tmem_writes[ts] = (it, 1)
        else:
            tmem_writes[ts] = (it, n + 1)

    def epilogue(w):
        for j in range(n_tiles):
            buf = j & 1
            yield wait(acc_full[buf], (j >> 1) & 1, j >> 1)
            assert acc_done[buf] == nkb, "epilogue read an accumulator before its MMAs completed"
            bufs.release(("acc", buf))
            acc_empty[buf].arrive()

    roles = {"tma": producer(), "mma": mma()}
    roles.update({f"dec{w}": decoder(w) for w in range(dec_warps)})
    roles.update({f"epi{w}": epilogue(w) for w in range(4)})
    return roles, q


KB = 1024
# k-block buffer sizes (weight boxes + token terms): a 16-row expert tile of the gate/up
# GEMM (36 KB), of the down GEMM (20 KB), a full 128-row gate/up tile (64 KB), a paired
# dense tile of 256 single-term rows (64 KB), a two-term one (96 KB)
GEMM_CASES = [
    ([36 * KB] * 3, 1, 200 * KB), ([36 * KB, 64 * KB, 36 * KB, 20 * KB], 5, 200 * KB),
    ([20 * KB] * 5, 4, 200 * KB), ([64 * KB] * 4, 32, 200 * KB), ([96 * KB] * 2, 6, 200 * KB),
    ([36 * KB, 44 * KB, 64 * KB, 52 * KB, 36 * KB, 20 * KB, 28 * KB], 3, 200 * KB),
    ([64 * KB, 36 * KB], 7, 64 * KB),      # one k-block in flight at a time
    ([4 * KB] * 3, 40, 200 * KB),           # more k-blocks than barrier pairs fit
]


@pytest.mark.parametrize("tile_bytes,nkb,cap", GEMM_CASES)
@pytest.mark.parametrize("nbuf", [2, 1])
def test_bf16_gemm_protocol(tile_bytes, nkb, cap, nbuf):
    for seed in range(30):
        roles, q = bf16_gemm(tile_bytes, nkb, cap, nbuf=nbuf)
        run(roles, q, seed, end_check=True)


def test_the_checker_catches_a_ring_without_the_footprint_check():
    """A producer that counts barrier pairs but not bytes overwrites a buffer still read."""
    caught = 0
    for seed in range(60):
        roles, q = bf16_gemm([36 * KB, 64 * KB, 20 * KB], 6, 128 * KB, bug="no_footprint_check")
        try:
            run(roles, q, seed, end_check=True)
        except AssertionError:
            caught += 1
    assert caught > 0


@pytest.mark.parametrize("n_tiles,nkb,stages", [(1, 1, 2), (3, 1, 6), (2, 5, 3), (5, 4, 6), (3, 16, 6), (6, 3, 2),
                                                (4, 7, 8)])
def test_lowp_gemm_protocol(n_tiles, nkb, stages):
    for seed in range(30):
        roles, q = lowp_gemm(n_tiles, nkb, stages)
        run(roles, q, seed, end_check=True)


def _lowp_with_count(f_empty_count, seed):
    orig = Barrier.__init__

    def patched(self, name, count):
        orig(self, name, f_empty_count if name.startswith("f_empty") else count)
    Barrier.__init__ = patched
    try:
        roles, q = lowp_gemm(3, 5, 2, dec_warps=8)
    finally:
        Barrier.__init__ = orig
    run(roles, q, seed)


def test_the_checker_catches_a_wrong_count():
    """With f_empty counting the decoder warps only (the MMAs' release of the token tiles
    not awaited), some interleaving must be reported: a stage overwritten while read, a
    release without a reader, a barrier run past its waiter, or a deadlock."""
    caught = 0
    for seed in range(100):
        try:
            _lowp_with_count(8, seed)
        except AssertionError:
            caught += 1
    assert caught > 0
    for seed in range(20):       # and the kernel's count passes the same interleavings
        _lowp_with_count(9, seed)


# ---------------------------------------------------------------- the single-head attention kernel (k_tc_attn.cu)

def two_ring_plan(nck, cur_from, kslots, vslots):
    """The single-head kernel's rings: chunk j's K parts (two for own keys) take the next
    entries of a ring of `kslots` half-slots, its V^T parts those of a ring of `vslots`
    half-slots numbered after the K ring's; returns [(K parts, V parts)], each part
    (half-slot, its use index)."""
    ek = ev = 0
    plan = []
    for j in range(nck):
        n = 2 if j >= cur_from else 1
        kp = [((ek + i) % kslots, (ek + i) // kslots) for i in range(n)]
        vp = [(kslots + (ev + i) % vslots, (ev + i) // vslots) for i in range(n)]
        plan.append((kp, vp))
        ek += n
        ev += n
    return plan


def attention(nck, seed, cur_from=None, kslots=3, vslots=2, n_warps=4, flags=None, give_up_at=None, drain=True,
              load_drain=True, bug=None, shared_ring=False):
    """tc_attn_kernel's hand-offs (128-key chunks, two S buffers, one P buffer): one load
    thread fills the query tile, then each chunk's K into a ring of `kslots` half-slots,
    another each chunk's V^T into a ring of `vslots` (shared_ring: one ring of kslots +
    vslots half-slots for both, K then V^T per chunk, filled by one load thread -- which
    the two issuing threads cannot share, see below).
    Two issuing threads: the S thread issues S(j) into S buffer j & 1 once chunk j's K has
    landed and the softmax warps have read S(j - 2) (s_free), then a commit freeing the K
    half-slots; the PV thread issues PV(j) once chunk j's V^T has landed and P(j) is
    written, then a commit freeing the V^T half-slots; their completions interleave in any
    order, each thread's in its own issue order.  Each softmax warp reads S(j) and signals
    s_free, then -- once PV(j - 1) is complete (O stable, P read) -- maybe rescales O,
    writes P(j) and signals.  Chunks [cur_from, nck) are the call's own (two half-slots per
    operand).  Every role reaches the exit barrier; both issuing threads drain their
    commits (`drain`), and after an abort the load warp waits for the loads it issued
    (`load_drain`).

    bug: "no_s_free_wait" -- S(j) issued without waiting for the softmax's read of S(j - 2);
    "no_pv_wait" -- P(j) written without waiting for PV(j - 1).
    flags / give_up_at: abort mode as in attention_two_heads below."""
    rng = random.Random(seed * 7919 + nck)
    cf = nck if cur_from is None else cur_from
    slots = kslots + vslots
    plan = half_slot_plan(nck, cf, slots) if shared_ring else two_ring_plan(nck, cf, kslots, vslots)
    q_bar = Barrier("q", 1)
    hs_full = [Barrier(f"hs_full{s}", 1) for s in range(slots)]
    hs_free = [Barrier(f"hs_free{s}", 1) for s in range(slots)]
    s_full = [Barrier(f"s_full{b}", 1) for b in range(2)]
    s_free = [Barrier(f"s_free{b}", n_warps) for b in range(2)]
    p_ready, pv_done = Barrier("p_ready", n_warps), Barrier("pv_done", 1)
    drain_bar = Barrier("drain", 2)
    exit_bar = Barrier("exit", n_warps + 4)            # the __syncthreads every role reaches at the end
    bufs, q = Buffers(), AsyncPerThread(2)
    st = dict(pv_issued=0, pv_done=0)
    p_writes = {}
    steps = [0]
    uses = {}                                          # half-slot -> use index last loaded into it

    def bw(bar, parity, phase):
        if flags is None:
            return wait(bar, parity, phase)
        steps[0] += 1
        if steps[0] == give_up_at:
            flags["abort"] = True
        return ("waitab", bar, parity, phase)

    def passed(bar, parity):
        return flags is None or (bar.completed % 2) != parity

    def load(parts_of, with_q):
        """A load thread: the ring entries parts_of(j) of each chunk, in order."""
        if with_q:
            q_bar.arrive_expect_tx(64)
            q.loads.append(lambda: q_bar.complete_tx(64))
        loaded = {}
        ok = True
        for j in range(nck):
            for x, u in parts_of(j):
                if u >= 1:
                    yield bw(hs_free[x], (u - 1) & 1, u - 1)
                    if not passed(hs_free[x], (u - 1) & 1):
                        ok = False
                        break
                bufs.fill(("hs", x), 1)                 # K: read by S(j); V^T: by PV(j)
                uses[x] = u
                hs_full[x].arrive_expect_tx(32)
                q.loads.append(lambda x=x: hs_full[x].complete_tx(32))
                loaded[x] = loaded.get(x, 0) + 1
            if not ok:
                break
        # the kernel decides on the wind-down after every role has reached the exit barrier
        exit_bar.arrive()
        yield wait(exit_bar, 0, 0)
        if flags is not None and flags["abort"] and load_drain:
            if with_q:
                yield wait(q_bar, 0, None)
            for x, n in loaded.items():
                yield wait(hs_full[x], (n - 1) & 1, None)

    def leaving(body):
        """A role that reaches the exit barrier however its body ends."""
        try:
            yield from body
        finally:
            exit_bar.arrive()

    def s_thread():
        mq = q.by[0]
        yield bw(q_bar, 0, 0)
        ok = passed(q_bar, 0)
        for j in range(nck if ok else 0):
            b = j & 1
            for x, u in plan[j][0]:
                yield bw(hs_full[x], u & 1, u)
                if not passed(hs_full[x], u & 1):
                    ok = False
                    break
                assert uses.get(x) == u and hs_full[x].completed == u + 1, f"S({j}) read half-slot {x} before use {u} landed"
            if ok and j >= 2 and bug != "no_s_free_wait":
                yield bw(s_free[b], ((j - 2) >> 1) & 1, (j - 2) >> 1)
                ok = passed(s_free[b], ((j - 2) >> 1) & 1)
            if not ok:
                break
            for w in range(n_warps):                   # S(j): each softmax warp reads its 32 lanes
                bufs.fill(("S", b, w), 1)

            def s_done(j=j, b=b):
                for x, _ in plan[j][0]:
                    bufs.release(("hs", x))
                s_full[b].arrive()
            mq.append(s_done)
            for x, _ in plan[j][0]:
                mq.append(lambda x=x: hs_free[x].arrive())
        if drain:
            mq.append(lambda: drain_bar.arrive())
            yield wait(drain_bar, 0, 0)

    def pv_thread():
        mq = q.by[1]
        for i in range(nck):
            ok = True
            for x, u in plan[i][1]:
                yield bw(hs_full[x], u & 1, u)
                if not passed(hs_full[x], u & 1):
                    ok = False
                    break
                assert uses.get(x) == u and hs_full[x].completed == u + 1, f"PV({i}) read half-slot {x} before use {u} landed"
            if not ok:
                break
            yield bw(p_ready, i & 1, i)
            if not passed(p_ready, i & 1):
                break
            assert p_writes.get("p") == (i, n_warps), "PV read a P not fully written"
            st["pv_issued"] += 1

            def fin(i=i):
                st["pv_done"] += 1
                for w in range(n_warps):
                    bufs.release(("p", w))
                for x, _ in plan[i][1]:
                    bufs.release(("hs", x))
                pv_done.arrive()
            mq.append(fin)
            for x, _ in plan[i][1]:
                mq.append(lambda x=x: hs_free[x].arrive())
        if drain:
            mq.append(lambda: drain_bar.arrive())

    def softmax(w):
        for j in range(nck):
            b = j & 1
            yield bw(s_full[b], (j >> 1) & 1, j >> 1)
            if not passed(s_full[b], (j >> 1) & 1):
                return
            bufs.release(("S", b, w))                  # this warp's lanes of S(j) read into registers
            s_free[b].arrive()
            if j > 0 and bug != "no_pv_wait":
                yield bw(pv_done, (j - 1) & 1, j - 1)
                if not passed(pv_done, (j - 1) & 1):
                    return
                if rng.random() < 0.4:                 # some row's max grew: O is rescaled here
                    assert st["pv_done"] >= j and st["pv_issued"] <= j, "O rescaled while a PV may write it"
            bufs.fill(("p", w), 1)                     # this warp's lanes of P(j), read by PV(j)
            last, n = p_writes.get("p", (None, 0))
            p_writes["p"] = (j, 1) if last != j else (j, n + 1)
            p_ready.arrive()
        yield bw(pv_done, (nck - 1) & 1, nck - 1)
        if passed(pv_done, (nck - 1) & 1):
            assert st["pv_done"] == nck

    if shared_ring:
        roles = {"load": load(lambda j: plan[j][0] + plan[j][1], True), "load_idle": leaving(iter(()))}
    else:
        roles = {"load_k": load(lambda j: plan[j][0], True), "load_v": load(lambda j: plan[j][1], False)}
    roles.update({"mma_s": leaving(s_thread()), "mma_pv": leaving(pv_thread())})
    roles.update({f"sm{w}": leaving(softmax(w)) for w in range(n_warps)})
    return roles, q


@pytest.mark.parametrize("nck,cur_from", [(1, 1), (1, 0), (2, 2), (2, 1), (2, 0), (3, 3), (4, 2), (5, 3), (6, 0),
                                          (7, 5), (9, 9), (12, 10)])
def test_attention_protocol(nck, cur_from):
    """No deadlock, no overrun, no half-slot, S or P buffer refilled while read, no P read
    before all its writers, no O rescaled under a PV, nothing in flight when the CTA leaves."""
    for seed in range(30):
        roles, q = attention(nck, seed, cur_from=cur_from)
        run(roles, q, seed, end_check=True)


@pytest.mark.parametrize("bug", ["no_s_free_wait", "no_pv_wait"])
def test_attention_protocol_catches_its_planted_mistakes(bug):
    """S(j) issued before the softmax has read S(j - 2) from the same buffer, or P(j)
    written before PV(j - 1) has read P(j - 1): some interleaving overwrites a buffer
    still read."""
    caught = 0
    for seed in range(60):
        roles, q = attention(6, seed, cur_from=4, bug=bug)
        try:
            run(roles, q, seed, end_check=True)
        except AssertionError as e:
            caught += any(m in str(e) for m in ("overwritten", "PV read", "rescaled", "deadlock"))
    assert caught > 0


def test_attention_with_one_shared_ring_reads_a_half_slot_too_early():
    """One ring for K and V^T with two issuing threads: the S thread can reach a K entry whose
    half-slot still waits for an earlier V^T use to land, and its parity wait passes at once
    (a phase behind looks like a completed one).  The separate rings exist for this."""
    caught = 0
    for seed in range(300):
        roles, q = attention(9, seed, cur_from=3, shared_ring=True)
        try:
            run(roles, q, seed, end_check=True)
        except AssertionError as e:
            caught += "before use" in str(e) or "released twice" in str(e) or "overwritten" in str(e)
    assert caught > 0


def test_attention_with_the_smallest_rings():
    """One half-slot per ring deadlocks on a chunk of own keys (two parts); two per ring do
    not."""
    with pytest.raises(AssertionError, match="deadlock"):
        roles, q = attention(4, 0, cur_from=2, kslots=1, vslots=1)
        run(roles, q, 0)
    for seed in range(20):
        roles, q = attention(6, seed, cur_from=2, kslots=2, vslots=2)
        run(roles, q, seed, end_check=True)


def test_attention_leaves_nothing_in_flight():
    """Without the issuing threads' drain some interleaving leaves a commit landing after
    the CTA is gone."""
    left = 0
    for seed in range(60):
        roles, q = attention(6, seed, cur_from=4, drain=False)
        try:
            run(roles, q, seed, end_check=True)
        except AssertionError as e:
            left += "pending" in str(e)
    assert left > 0


@pytest.mark.parametrize("nck,cur_from", [(4, 2), (7, 4), (6, 0), (3, 3)])
def test_attention_winds_down_after_a_timeout(nck, cur_from):
    """A bounded wait gives up at a random point: every role leaves and, with the load and
    MMA drains, nothing is in flight when they have."""
    for seed in range(150):
        rng = random.Random(seed)
        flags = {"abort": False}
        roles, q = attention(nck, seed, cur_from=cur_from, flags=flags, give_up_at=rng.randrange(1, 14 * nck))
        run_ab(roles, q, flags, seed, end_check=True)


# ---------------------------------------------------------------- the fused vocabulary/update GEMM (k_tc_vocab_update.cu)

def test_fused_vocab_epilogue_barriers():
    """Four warps meeting at a named barrier 2 + 2 * chunks times per tile, interleaved with
    the accumulator hand-offs: no deadlock and no phase overrun."""
    for n_tiles, nkb, stages, chunks in ((1, 2, 2, 1), (3, 4, 3, 16), (5, 2, 4, 3)):
        for seed in range(20):
            full = [Barrier(f"full{s}", 1) for s in range(stages)]
            empty = [Barrier(f"empty{s}", 1) for s in range(stages)]
            acc_full = [Barrier(f"acc_full{b}", 1) for b in range(2)]
            acc_empty = [Barrier(f"acc_empty{b}", 4) for b in range(2)]
            named = Barrier("bar1", 4)
            bufs, q = Buffers(), Async()
            acc_done = {}

            def producer():
                it = 0
                for t in range(n_tiles):
                    for kb in range(nkb):
                        s = it % stages
                        yield wait(empty[s], ((it // stages) & 1) ^ 1, it // stages - 1)
                        bufs.fill(("smem", s), 1)
                        full[s].arrive_expect_tx(64)
                        q.loads.append(lambda s=s: full[s].complete_tx(64))
                        it += 1

            def mma():
                it = 0
                for j in range(n_tiles):
                    buf = j & 1
                    yield wait(acc_empty[buf], ((j >> 1) & 1) ^ 1, (j >> 1) - 1)
                    bufs.fill(("acc", buf), 4)
                    acc_done[buf] = 0
                    for kb in range(nkb):
                        s = it % stages
                        yield wait(full[s], (it // stages) & 1, it // stages)

                        def done(s=s, buf=buf):
                            acc_done[buf] += 1
                            bufs.release(("smem", s))
                            empty[s].arrive()
                        q.mma.append(done)
                        it += 1
                    q.mma.append(lambda b=buf: acc_full[b].arrive())

            def epilogue(w):
                k = 0  # named-barrier phases this warp has passed

                def meet():
                    nonlocal k
                    named.arrive()
                    yield wait(named, k & 1, k)
                    k += 1
                for j in range(n_tiles):
                    buf = j & 1
                    yield wait(acc_full[buf], (j >> 1) & 1, j >> 1)
                    yield from meet()          # post the wait result
                    yield from meet()          # the vote is read; the flags may be rewritten
                    assert acc_done[buf] == nkb
                    for c in range(chunks):
                        yield from meet()      # the four warps' records are in shared memory
                        yield from meet()      # merged and stored; the next chunk may write
                    bufs.release(("acc", buf))
                    acc_empty[buf].arrive()

            roles = {"tma": producer(), "mma": mma()}
            roles.update({f"epi{w}": epilogue(w) for w in range(4)})
            run(roles, q, seed)


# ---------------------------------------------------------------- leaving on a timeout

def fused_epilogue_with_abort(n_tiles, nkb, stages, chunks, rng, vote=True):
    """The fused vocabulary/update kernel's roles where some wait gives up: a bounded
    mbarrier wait returns (false) once the CTA's abort flag is set, a named barrier does
    not.  With the vote, the four epilogue warps agree before every named barrier on
    whether to go on; without it, each warp leaves alone."""
    full = [Barrier(f"full{s}", 1) for s in range(stages)]
    empty = [Barrier(f"empty{s}", 1) for s in range(stages)]
    acc_full = [Barrier(f"acc_full{b}", 1) for b in range(2)]
    acc_empty = [Barrier(f"acc_empty{b}", 4) for b in range(2)]
    named = Barrier("bar1", 4)
    q = Async()
    flags = {"abort": False}
    epi_ok = [True] * 4
    give_up_at = rng.randrange(1, 2 * n_tiles * nkb + 2)   # the step at which some wait times out
    steps = [0]

    def wait_ab(bar, parity, phase):
        # a bounded wait: passes on the phase, or gives up once the abort flag is set (or
        # when this wait is the one chosen to time out, which raises the flag)
        steps[0] += 1
        if steps[0] == give_up_at:
            flags["abort"] = True
        return ("waitab", bar, parity, phase)

    def ok_after(bar, parity):
        return (bar.completed % 2) != parity

    drain_bar = Barrier("drain", 1)

    def producer():
        it = 0

        def issue_all():
            nonlocal it
            for t in range(n_tiles):
                for kb in range(nkb):
                    s = it % stages
                    par = ((it // stages) & 1) ^ 1
                    yield wait_ab(empty[s], par, None)
                    if not ok_after(empty[s], par):
                        return
                    full[s].arrive_expect_tx(64)
                    q.loads.append(lambda s=s: full[s].complete_tx(64))
                    it += 1
        yield from issue_all()
        if flags["abort"]:                            # the wind-down: the newest load of every stage
            for i in range(max(0, it - stages), it):
                yield wait(full[i % stages], (i // stages) & 1, None)

    def mma():
        it = 0

        def issue_all():
            nonlocal it
            for j in range(n_tiles):
                buf = j & 1
                par = ((j >> 1) & 1) ^ 1
                yield wait_ab(acc_empty[buf], par, None)
                if not ok_after(acc_empty[buf], par):
                    return
                for kb in range(nkb):
                    s = it % stages
                    par2 = (it // stages) & 1
                    yield wait_ab(full[s], par2, None)
                    if not ok_after(full[s], par2):
                        return
                    q.mma.append(lambda s=s: empty[s].arrive())
                    it += 1
                q.mma.append(lambda b=buf: acc_full[b].arrive())
        yield from issue_all()
        q.mma.append(lambda: drain_bar.arrive())      # the final commit, waited for before the CTA leaves
        yield wait(drain_bar, 0, 0)

    def epilogue(w):
        k = 0

        def meet():
            nonlocal k
            named.arrive()
            yield wait(named, k & 1, k)
            k += 1
        for j in range(n_tiles):
            buf = j & 1
            par = (j >> 1) & 1
            yield wait_ab(acc_full[buf], par, None)
            ok = ok_after(acc_full[buf], par)
            if vote:
                epi_ok[w] = ok
                yield from meet()
                all_ok = all(epi_ok)
                yield from meet()
                if not all_ok:
                    return
            elif not ok:
                return
            for c in range(chunks):
                yield from meet()
                yield from meet()
            acc_empty[buf].arrive()

    roles = {"tma": producer(), "mma": mma()}
    roles.update({f"epi{w}": epilogue(w) for w in range(4)})
    return roles, q, flags


def run_ab(roles, q, flags, seed, max_steps=200000, end_check=False):
    """run() where an abort-aware wait also passes once the abort flag is set."""
    rng = random.Random(seed)
    blocked = {}
    live = dict(roles)
    for _ in range(max_steps):
        if not live:
            if end_check:
                assert not q, f"{len(q.loads)} loads and {len(q.mma)} MMA completions pending after the last role left"
            return
        ready = []
        for name in live:
            b = blocked.get(name)
            if b is None:
                ready.append(name)
            elif b[0] == "waitab" and (flags["abort"] or (b[1].completed % 2) != b[2]):
                ready.append(name)
            elif b[0] == "wait" and b[1].passes(b[2], b[3]):
                ready.append(name)
        choices = ready + (["<async>"] if q else [])
        assert choices, f"deadlock: blocked {sorted((n, b[1].name) for n, b in blocked.items())}"
        pick = rng.choice(choices)
        if pick == "<async>":
            q.step(rng)
            continue
        blocked.pop(pick, None)
        try:
            step = next(live[pick])
        except StopIteration:
            del live[pick]
            continue
        if step is not None:
            blocked[pick] = step
    raise AssertionError("no progress")


def test_fused_epilogue_warps_leave_together_on_a_timeout():
    """With the vote every role of the fused kernel finishes whichever wait gives up (the
    final __syncthreads is reached); without it some interleaving leaves warps blocked at
    the named barrier for good -- the hang the vote prevents."""
    for seed in range(300):
        rng = random.Random(seed)
        roles, q, flags = fused_epilogue_with_abort(3, 3, 2, 2, rng, vote=True)
        run_ab(roles, q, flags, seed, end_check=True)
    hung = 0
    for seed in range(300):
        rng = random.Random(seed)
        roles, q, flags = fused_epilogue_with_abort(3, 3, 2, 2, rng, vote=False)
        try:
            run_ab(roles, q, flags, seed)
        except AssertionError as e:
            hung += "deadlock" in str(e)
    assert hung > 0


# ---------------------------------------------------------------- the attention redesign (on paper)

def half_slot_plan(nck, cur_from, slots):
    """The head-pair kernel's ring: chunk j takes the next one half-slot (cached keys) or
    two (own keys: hi and lo parts) for its K, then as many for its V^T; returns
    [(K parts, V parts)], each part (half-slot, its use index)."""
    nxt, uses, plan = 0, [0] * slots, []
    for j in range(nck):
        n = 2 if j >= cur_from else 1
        parts = []
        for _ in range(2):
            lst = []
            for _ in range(n):
                lst.append((nxt, uses[nxt]))
                uses[nxt] += 1
                nxt = (nxt + 1) % slots
            parts.append(lst)
        plan.append(tuple(parts))
    return plan


class AsyncPerThread(Async):
    """Completions of several issuing threads: each thread's MMAs and commits complete in its
    own issue order, the threads' streams interleave in any order."""

    def __init__(self, n):
        super().__init__()
        self.by = [[] for _ in range(n)]

    def __bool__(self):
        return bool(self.loads or any(self.by))

    def step(self, rng):
        busy = [q for q in self.by if q]
        if busy and (not self.loads or rng.random() < 0.5):
            rng.choice(busy).pop(0)()
        else:
            self.loads.pop(rng.randrange(len(self.loads)))()


def attention_two_heads(nck, seed, slots=3, warps_per_head=4, cur_from=None, flags=None, give_up_at=None,
                        drain=True, load_drain=True, bug=None):
    """The head-pair attention kernel's hand-offs (128-key chunks): a load warp fills a ring
    of `slots` half-slots, each chunk's K then its V^T; one MMA thread per head issues, per
    chunk, its S(j) -- once its PV(j-1) has completed, since S overwrites the head's one
    S/P region -- and a commit towards freeing the K half-slots, then its PV(j) once its
    softmax warps have written P(j), and a commit towards freeing the V half-slots; a
    half-slot's free barrier counts one commit per head.  Each head's softmax warps read
    S(j), maybe rescale O (after PV(j-1)), write P over S and signal.  Each MMA thread
    drains its commits before the CTA leaves (`drain`).

    bug: "no_pv_wait" -- S(j) issued without waiting for PV(j-1); "free_count_one" -- the
    half-slots' free barriers count one commit, so the first head's frees the slot.

    flags: abort mode -- every bounded wait also passes once flags["abort"] is set, the
    give_up_at-th wait raises it (a timeout), a role whose wait failed leaves its loop,
    and the load warp then waits for the loads it issued (`load_drain`)."""
    rng = random.Random(seed * 104729 + nck)
    plan = half_slot_plan(nck, nck if cur_from is None else cur_from, slots)
    H = 2
    free_count = 1 if bug == "free_count_one" else H
    hs_full = [Barrier(f"hs_full{s}", 1) for s in range(slots)]
    hs_free = [Barrier(f"hs_free{s}", free_count) for s in range(slots)]
    drain_bar = Barrier("drain", H)
    s_full = [Barrier(f"s_full{h}", 1) for h in range(H)]
    p_ready = [Barrier(f"p_ready{h}", warps_per_head) for h in range(H)]
    pv_done = [Barrier(f"pv_done{h}", 1) for h in range(H)]
    bufs, q = Buffers(), AsyncPerThread(H)
    st = {"pv_done": [0, 0], "pv_issued": [0, 0]}
    p_writes = {}
    steps = [0]
    uses = {}                                         # half-slot -> use index last loaded into it

    def bw(bar, parity, phase):
        """A bounded wait (abort-aware in abort mode)."""
        if flags is None:
            return wait(bar, parity, phase)
        steps[0] += 1
        if steps[0] == give_up_at:
            flags["abort"] = True
        return ("waitab", bar, parity, phase)

    def passed(bar, parity):
        return flags is None or (bar.completed % 2) != parity

    def load():
        loaded = [0] * slots
        ok = True
        for j in range(nck):
            for parts in plan[j]:
                for s, u in parts:
                    if u >= 1:
                        yield bw(hs_free[s], (u - 1) & 1, u - 1)
                        if not passed(hs_free[s], (u - 1) & 1):
                            ok = False
                            break
                    bufs.fill(("hs", s), H)           # K: both heads' S read it; V^T: both PVs
                    uses[s] = u
                    hs_full[s].arrive_expect_tx(32)
                    q.loads.append(lambda s=s: hs_full[s].complete_tx(32))
                    loaded[s] += 1
                if not ok:
                    break
            if not ok:
                break
        if flags is not None and flags["abort"] and load_drain:
            for s in range(slots):                    # the wind-down: the last load of each half-slot
                if loaded[s]:
                    yield wait(hs_full[s], (loaded[s] - 1) & 1, None)

    def mma(h):
        mq = q.by[h]
        ok = True
        for j in range(nck):
            k_parts, v_parts = plan[j]
            for x, u in k_parts:
                yield bw(hs_full[x], u & 1, u)
                if not passed(hs_full[x], u & 1):
                    ok = False
                    break
                assert uses.get(x) == u and hs_full[x].completed == u + 1, f"S read half-slot {x} before use {u} landed"
            if ok and j >= 1 and bug != "no_pv_wait":
                yield bw(pv_done[h], (j - 1) & 1, j - 1)
                ok = passed(pv_done[h], (j - 1) & 1)
            if not ok:
                break
            for w in range(warps_per_head):           # S: each warp reads its own 32 lanes
                bufs.fill(("sp", h, w), 1)

            def s_done(h=h, j=j):
                for x, _ in plan[j][0]:
                    bufs.release(("hs", x))
                s_full[h].arrive()
            mq.append(s_done)
            for x, _ in k_parts:                      # this head's commit per K half-slot
                mq.append(lambda x=x: hs_free[x].arrive())
            for x, u in v_parts:
                yield bw(hs_full[x], u & 1, u)
                if not passed(hs_full[x], u & 1):
                    ok = False
                    break
                assert uses.get(x) == u and hs_full[x].completed == u + 1, f"PV read half-slot {x} before use {u} landed"
            if not ok:
                break
            yield bw(p_ready[h], j & 1, j)
            if not passed(p_ready[h], j & 1):
                break
            assert p_writes.get(h) == (j, warps_per_head), "PV read a P not fully written"
            st["pv_issued"][h] += 1

            def pv_fin(h=h, j=j):
                st["pv_done"][h] += 1
                for w in range(warps_per_head):       # every warp's lanes of P(j) were read
                    bufs.release(("sp", h, w))
                for x, _ in plan[j][1]:
                    bufs.release(("hs", x))
                pv_done[h].arrive()
            mq.append(pv_fin)
            for x, _ in v_parts:                      # this head's commit per V^T half-slot
                mq.append(lambda x=x: hs_free[x].arrive())
        if drain:                                     # every commit issued above has landed
            mq.append(lambda: drain_bar.arrive())
            if h == 0:
                yield wait(drain_bar, 0, 0)

    def softmax(h, w):
        for j in range(nck):
            yield bw(s_full[h], j & 1, j)
            if not passed(s_full[h], j & 1):
                return
            bufs.release(("sp", h, w))                # this warp's lanes of S read into registers
            if j > 0 and rng.random() < 0.4:          # the row max grew: rescale O after PV(j-1)
                yield bw(pv_done[h], (j - 1) & 1, j - 1)
                if not passed(pv_done[h], (j - 1) & 1):
                    return
                assert st["pv_done"][h] >= j and st["pv_issued"][h] <= j, "O rescaled while a PV may write it"
            bufs.fill(("sp", h, w), 1)                # P over this warp's lanes of S, read by PV(j)
            last, n = p_writes.get(h, (None, 0))
            p_writes[h] = (j, 1) if last != j else (j, n + 1)
            p_ready[h].arrive()
        yield bw(pv_done[h], (nck - 1) & 1, nck - 1)
        if passed(pv_done[h], (nck - 1) & 1):
            assert st["pv_done"][h] == nck

    roles = {"load": load()}
    for h in range(H):
        roles[f"mma{h}"] = mma(h)
        roles.update({f"sm{h}{w}": softmax(h, w) for w in range(warps_per_head)})
    return roles, q


@pytest.mark.parametrize("nck,cur_from", [(1, 1), (1, 0), (2, 2), (3, 3), (4, 2), (7, 7), (7, 4), (12, 8), (6, 0)])
def test_head_pair_attention_protocol(nck, cur_from):
    """Cached chunks in one half-slot per operand, the call's own (current) chunks in two:
    no deadlock, no overrun, no buffer refilled while read, no P read before all its
    writers, no O rescaled under a PV."""
    for seed in range(40):
        roles, q = attention_two_heads(nck, seed, cur_from=cur_from)
        run(roles, q, seed, end_check=True)


@pytest.mark.parametrize("bug", ["no_pv_wait", "free_count_one"])
def test_head_pair_attention_protocol_catches_its_planted_mistakes(bug):
    """S(j) issued before PV(j-1) has read P(j-1) from the same TMEM region, or a half-slot
    freed by the first head's commit before the other head's MMAs read it: some
    interleaving overwrites a buffer that is still read."""
    caught = 0
    for seed in range(80):
        roles, q = attention_two_heads(6, seed, cur_from=4, bug=bug)
        try:
            run(roles, q, seed, end_check=True)
        except AssertionError:
            caught += 1
    assert caught > 0


def test_head_pair_attention_leaves_nothing_in_flight():
    """When the last role leaves, no MMA completion or commit may still be pending (it would
    arrive on released shared memory): the MMA warp's drain makes that hold in every
    interleaving; without it some interleaving leaves a commit behind."""
    for seed in range(60):
        roles, q = attention_two_heads(6, seed, cur_from=4)
        run(roles, q, seed, end_check=True)
    left = 0
    for seed in range(60):
        roles, q = attention_two_heads(6, seed, cur_from=4, drain=False)
        try:
            run(roles, q, seed, end_check=True)
        except AssertionError as e:
            left += "pending" in str(e)
    assert left > 0


@pytest.mark.parametrize("nck,cur_from", [(4, 2), (7, 4), (6, 0)])
def test_head_pair_attention_winds_down_after_a_timeout(nck, cur_from):
    """A bounded wait gives up at a random point: every role leaves (no deadlock), and with
    the load warp's drain and the MMA warp's drain nothing is in flight when they have.
    Without the load drain, some timeout leaves a load landing after the CTA is gone."""
    for seed in range(150):
        rng = random.Random(seed)
        flags = {"abort": False}
        roles, q = attention_two_heads(nck, seed, cur_from=cur_from, flags=flags,
                                       give_up_at=rng.randrange(1, 12 * nck))
        run_ab(roles, q, flags, seed, end_check=True)
    left = 0
    for seed in range(150):
        rng = random.Random(seed)
        flags = {"abort": False}
        roles, q = attention_two_heads(nck, seed, cur_from=cur_from, flags=flags,
                                       give_up_at=rng.randrange(1, 12 * nck), load_drain=False)
        try:
            run_ab(roles, q, flags, seed, end_check=True)
        except AssertionError as e:
            left += "pending" in str(e)
    assert left > 0
