"""CPU models of the mbarrier protocols of the two pipelined kernels.

An mbarrier wait by phase parity passes when the phase with that parity is
the last completed one, so a waiter that falls two phases behind would pass
on the wrong phase. These models replay every role of a CTA (producers, MMA
issuer, consumer / softmax warps) as coroutines over counting barriers. TMA
landings, MMA completions and the order in which roles run are drawn at
random. They check that no run deadlocks and that every wait names the
phase just completed, never an older one. They also check the buffer rules:
a tile is read only after it landed, S is overwritten only after it was
read and its P consumed, and the tail V rows are zeroed before any P.V
reads them.

The models restate the protocols of pa_decode.cuh (decode ring; the
broadcast ring of the shared-prefix kernels, also used by the mma.sync
prefill in pa_prefill.cuh) and pa_prefill.cuh (tcgen05 prefill); they do
not run the kernels.
"""
import random

import pytest


# --------------------------------------------------------------- decode ring

def _decode_ring_false_pass(nblk, warps, stages, seed):
    """One head, `warps` consumer warps taking blocks w, w + W, ... from
    stage i % stages. The wait is by parity, so a wait passes when the
    stage's phase count has the other parity. Returns True if a consumer
    passed its wait before its block had landed."""
    rnd = random.Random(seed)
    full = [0] * stages
    empty = [0] * stages
    empty_cnt = [0] * stages
    landed, inflight = set(), []
    nxt = 0
    cons = list(range(warps))
    for _ in range(100000):
        acts = []
        if nxt < nblk:
            s, use = nxt % stages, nxt // stages
            if use == 0 or (empty[s] & 1) != ((use - 1) & 1):
                acts.append(("prod",))
        if inflight:
            acts.append(("land",))
        for w, i in enumerate(cons):
            if i < nblk and (full[i % stages] & 1) != ((i // stages) & 1):
                acts.append(("cons", w))
        if not acts:
            return False
        a = rnd.choice(acts)
        if a[0] == "prod":
            inflight.append(nxt)
            nxt += 1
        elif a[0] == "land":
            b = inflight.pop(rnd.randrange(len(inflight)))
            landed.add(b)
            full[b % stages] += 1
        else:
            i = cons[a[1]]
            if i not in landed:
                return True
            s = i % stages
            empty_cnt[s] += 1
            if empty_cnt[s] == 1:
                empty_cnt[s] = 0
                empty[s] += 1
            cons[a[1]] += warps
    return False


@pytest.mark.parametrize("warps", [1, 2, 4])
def test_decode_ring_is_sound_when_warps_divide_stages(warps):
    for stages in range(warps, 9, warps):
        for nblk in (1, 3, 5, 8, 13, 30):
            for seed in range(25):
                assert not _decode_ring_false_pass(nblk, warps, stages, seed), (warps, stages, nblk, seed)


def test_decode_ring_false_passes_without_the_rule():
    # the reason the library rejects stages % warps_per_head != 0
    found = set()
    for warps, stages in [(2, 3), (4, 2), (4, 6)]:
        for nblk in (8, 13, 30):
            for seed in range(60):
                if _decode_ring_false_pass(nblk, warps, stages, seed):
                    found.add((warps, stages))
    assert found == {(2, 3), (4, 2), (4, 6)}


# ------------------------------------------------------------ broadcast ring

def _broadcast_ring_run(ntiles, consumers, stages, seed, release_count=None):
    """The ring of the shared-prefix kernels and the mma.sync prefill: one
    producer puts tile j into stage j % stages once every consumer has
    released the stage's previous tile (the empty barrier counts
    `consumers` arrivals); every consumer warp reads every tile in order,
    waiting on the stage's full barrier by parity. Landings and the order of
    the roles are random. Returns a description of the first violation, or
    None. `release_count` replaces the empty barrier's arrival count (to
    plant a mistake)."""
    rnd = random.Random(seed)
    release_count = consumers if release_count is None else release_count
    full = [0] * stages            # completed phases
    empty = [0] * stages
    empty_cnt = [0] * stages
    content = [None] * stages      # tile held by each stage
    readers = [set() for _ in range(stages)]   # consumers between their wait and their release
    inflight = []
    nxt = 0
    cons = [0] * consumers         # next tile of each consumer
    holding = [None] * consumers   # stage a consumer has passed the wait on and not yet released
    for _ in range(200000):
        acts = []
        if nxt < ntiles:
            st, use = nxt % stages, nxt // stages
            if use == 0 or (empty[st] & 1) != ((use - 1) & 1):
                acts.append(("prod",))
        if inflight:
            acts.append(("land",))
        for c in range(consumers):
            if holding[c] is not None:
                acts.append(("release", c))
            elif cons[c] < ntiles:
                i = cons[c]
                if (full[i % stages] & 1) != ((i // stages) & 1):
                    acts.append(("read", c))
        if not acts:
            done = nxt == ntiles and not inflight and all(i == ntiles for i in cons)
            return None if done else "deadlock"
        a = rnd.choice(acts)
        if a[0] == "prod":
            inflight.append(nxt)
            nxt += 1
        elif a[0] == "land":
            j = inflight.pop(rnd.randrange(len(inflight)))
            st = j % stages
            if readers[st]:
                return f"tile {j} overwrote stage {st} while consumers {sorted(readers[st])} read it"
            content[st] = j
            full[st] += 1
        elif a[0] == "read":
            c = a[1]
            i = cons[c]
            st = i % stages
            if content[st] != i:
                return f"consumer {c} passed its wait for tile {i} but stage {st} holds {content[st]}"
            readers[st].add(c)
            holding[c] = st
        else:
            c = a[1]
            st = holding[c]
            readers[st].discard(c)
            holding[c] = None
            cons[c] += 1
            empty_cnt[st] += 1
            if empty_cnt[st] == release_count:
                empty_cnt[st] = 0
                empty[st] += 1
    return "no termination"


@pytest.mark.parametrize("consumers", [1, 2, 4])
def test_broadcast_ring_is_sound(consumers):
    for stages in (2, 3, 4, 6, 8):
        for ntiles in (1, 2, 5, 9, 17, 40):
            for seed in range(20):
                assert _broadcast_ring_run(ntiles, consumers, stages, seed) is None, \
                    (consumers, stages, ntiles, seed)


def test_broadcast_ring_model_catches_a_missing_release_count():
    # an empty barrier that completes on every arrival (count 1 instead of
    # `consumers`) lets the producer overwrite a stage a slower warp is still
    # reading, or a warp pass a stale phase: the model must report it
    found = [_broadcast_ring_run(17, 4, 2, seed, release_count=1) or "" for seed in range(40)]
    assert any(r.startswith("tile") and "overwrote" in r for r in found)


# ------------------------------------------------------- tcgen05 prefill

K_STAGES, V_STAGES = 3, 2


class _Bar:
    def __init__(self, name, count):
        self.name, self.count, self.pending, self.done = name, count, count, 0

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0, self.name
        if self.pending == 0:
            self.done += 1
            self.pending = self.count


def _prefill_run(n_kv, tail, seed):
    """One CTA of paged_prefill_tc_kernel: K and V producers, the MMA issuer
    and the eight softmax warps (pairs exchange their maxima every tile)."""
    rnd = random.Random(seed)
    bars = {}

    def mk(name, count):
        bars[name] = _Bar(name, count)

    mk("q", 8)
    for s in range(K_STAGES):
        mk(f"fk{s}", 1)
        mk(f"ek{s}", 1)
    for s in range(V_STAGES):
        mk(f"fv{s}", 1)
        mk(f"ev{s}", 1)
    for b in range(2):
        mk(f"sf{b}", 1)
        mk(f"sr{b}", 8)
    mk("pf", 8)
    mk("or", 1)
    for q in range(4):
        for par in range(2):
            mk(f"pair{q}{par}", 2)
        mk(f"pend{q}", 2)
    st = {"k": [None] * K_STAGES, "v": [None] * V_STAGES, "S": [None, None], "Sread": [set(), set()],
          "pv": set(), "zeroed": set()}
    pending = []

    def wait(b, k):
        return ("wait", b, k)

    def producer(kind, stages):
        for j in range(n_kv):
            s, use = j % stages, j // stages
            if use > 0:
                yield wait(f"e{kind}{s}", use - 1)
            pending.append((kind, j, s))
            yield ("nop",)

    def mma():
        yield wait("q", 0)

        def pv(i):
            yield wait("pf", i)
            yield wait(f"fv{i % V_STAGES}", i // V_STAGES)
            assert st["v"][i % V_STAGES] == i
            pending.append(("pv", i))
            yield ("nop",)

        for j in range(n_kv):
            yield wait(f"fk{j % K_STAGES}", j // K_STAGES)
            assert st["k"][j % K_STAGES] == j
            if j >= 2:
                yield wait(f"sr{j & 1}", (j - 2) // 2)
                yield wait("or", j - 2)          # P_{j-2} in this S buffer consumed
                assert (j - 2) in st["pv"]
            pending.append(("s", j))
            yield ("nop",)
            if j >= 1:
                yield from pv(j - 1)
        yield from pv(n_kv - 1)

    rescale = {j: rnd.random() < 0.3 for j in range(n_kv)}

    def softmax(w):
        q = w & 3
        yield ("arrive", "q")
        for j in range(n_kv):
            yield wait(f"sf{j & 1}", j // 2)
            assert st["S"][j & 1] == j
            yield ("arrive", f"sr{j & 1}", w)
            yield ("arrive", f"pair{q}{j & 1}")
            yield wait(f"pair{q}{j & 1}", j // 2)
            if j >= 1 and rescale[j]:
                yield wait("or", j - 1)
                assert (j - 1) in st["pv"]
            if tail and j == n_kv - 1:
                yield wait(f"fv{j % V_STAGES}", j // V_STAGES)
                st["zeroed"].add((j, w))
            yield ("arrive", "pf")
        yield ("arrive", f"pend{q}")
        yield wait(f"pend{q}", 0)
        yield wait("or", n_kv - 1)

    roles = {"pk": producer("k", K_STAGES), "pv": producer("v", V_STAGES), "mma": mma(),
             **{f"w{w}": softmax(w) for w in range(8)}}
    cur = {k: None for k in roles}
    alive = set(roles)
    for _ in range(400000):
        if not alive and not pending:
            return
        progressed = False
        if pending and rnd.random() < 0.4:
            op = pending.pop(rnd.randrange(len(pending)))
            if op[0] == "k":
                st["k"][op[2]] = op[1]
                bars[f"fk{op[2]}"].arrive()
            elif op[0] == "v":
                st["v"][op[2]] = op[1]
                bars[f"fv{op[2]}"].arrive()
            elif op[0] == "s":
                j = op[1]
                prev = st["S"][j & 1]
                if prev is not None:
                    assert len(st["Sread"][j & 1]) == 8, "S overwritten before all warps read it"
                    assert prev in st["pv"], "S overwritten while its P was still to be read by P.V"
                st["S"][j & 1] = j
                st["Sread"][j & 1] = set()
                bars[f"sf{j & 1}"].arrive()
                bars[f"ek{j % K_STAGES}"].arrive()
            else:
                i = op[1]
                if tail and i == n_kv - 1:
                    assert len([1 for (jj, _) in st["zeroed"] if jj == i]) == 8, "P.V read the V tail before zeroing"
                st["pv"].add(i)
                bars[f"ev{i % V_STAGES}"].arrive()
                bars["or"].arrive()
            progressed = True
        order = list(alive)
        rnd.shuffle(order)
        for r in order:
            ev = cur[r]
            if ev is None:
                try:
                    ev = next(roles[r])
                except StopIteration:
                    alive.discard(r)
                    progressed = True
                    continue
                cur[r] = ev
            if ev[0] == "wait":
                b = bars[ev[1]]
                assert b.done <= ev[2] + 1, f"{r} waits {ev[1]} phase {ev[2]} with {b.done} phases done"
                if b.done >= ev[2] + 1:
                    cur[r] = None
                    progressed = True
            elif ev[0] == "arrive":
                bars[ev[1]].arrive()
                if ev[1].startswith("sr"):
                    st["Sread"][int(ev[1][2])].add(ev[2])
                cur[r] = None
                progressed = True
            else:
                cur[r] = None
                progressed = True
        assert progressed or pending, f"deadlock: {cur}"
    raise AssertionError("no termination")


@pytest.mark.parametrize("n_kv", [1, 2, 3, 4, 7])
@pytest.mark.parametrize("tail", [False, True])
def test_prefill_protocol(n_kv, tail):
    for seed in range(60):
        _prefill_run(n_kv, tail, seed)
