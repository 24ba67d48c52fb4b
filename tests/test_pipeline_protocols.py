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
ROW_SPLIT = 1                  # softmax warps sharing a row (1: a thread owns its whole row)


class _Bar:
    def __init__(self, name, count):
        self.name, self.count, self.pending, self.done = name, count, count, 0

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0, self.name
        if self.pending == 0:
            self.done += 1
            self.pending = self.count


S_BUFS = 3                     # S buffers in tensor memory (P of a tile overwrites its S)


MMA_ISSUERS = 1               # threads issuing the MMAs (2: one for S, one for P.V)


S_READ_BARRIER = False        # True: the S issuer also waits for "S read by every softmax warp"


def _prefill_run(n_kv, tail, seed, p_bars=S_BUFS, o_bars=S_BUFS, row_split=ROW_SPLIT, issuers=MMA_ISSUERS,
                 s_read_barrier=S_READ_BARRIER, skip_pv_wait=False, release_barriers=True):
    """One CTA of paged_prefill_tc_kernel: K and V producers, the MMA issuer
    and the softmax warps: row_split per tensor-memory lane quadrant (with
    more than one, the parts of a row exchange their maxima every tile
    through shared-memory slots chosen by tile parity).
    With one MMA issuer, S is computed one buffer ahead of need: S_0 ..
    S_{B-2} first, then per tile j, S_{j+B-1} (once its buffer is free)
    before P.V of j. With two, one thread issues every S (each once its
    buffer is free) and another every P.V; a thread's MMAs complete in its
    issue order, the two threads' in any interleaving.
    P barriers are indexed by tile % p_bars, P.V-done barriers by
    tile % o_bars. Without s_read_barrier, an S buffer is reused on the P.V
    of its previous tile alone (that P.V follows every warp's P, which each
    warp writes after reading S). skip_pv_wait plants a mistake: S reuses a
    buffer without waiting for that P.V. Without release_barriers the
    producers reuse a K stage on "S ready" of its previous tile (K stages
    and S buffers are both three) and a V stage on "P.V done" of its
    previous tile, instead of barriers of their own (a variant that measured
    slower on B200; the kernel has release barriers)."""
    rnd = random.Random(seed)
    bars = {}
    SB = S_BUFS
    N_SOFTMAX = 4 * row_split

    def mk(name, count):
        bars[name] = _Bar(name, count)

    mk("q", N_SOFTMAX)
    for s in range(K_STAGES):
        mk(f"fk{s}", 1)
        mk(f"ek{s}", 1)
    for s in range(V_STAGES):
        mk(f"fv{s}", 1)
        mk(f"ev{s}", 1)
    for b in range(SB):
        mk(f"sf{b}", 1)
        mk(f"sr{b}", N_SOFTMAX)
    for b in range(p_bars):
        mk(f"pf{b}", N_SOFTMAX)
    for b in range(o_bars):
        mk(f"or{b}", 1)                       # P.V of a tile of this index done
    for q in range(4):
        for par in range(2):
            mk(f"pair{q}{par}", row_split)
        mk(f"pend{q}", row_split)
    st = {"k": [None] * K_STAGES, "v": [None] * V_STAGES, "S": [None] * SB, "Sread": [set() for _ in range(SB)],
          "pv": set(), "zeroed": set(), "P": [0] * n_kv,
          # exchange slots: [lane quadrant][tile parity][half] -> tile whose maximum it holds
          "x": [[[None] * row_split for _ in range(2)] for _ in range(4)]}
    pending = []   # tile loads in flight: they land in any order
    mma_qs = {"s": [], "pv": []} if issuers == 2 else {"all": []}   # per issuing thread, in order
    q_s, q_pv = (mma_qs["s"], mma_qs["pv"]) if issuers == 2 else (mma_qs["all"], mma_qs["all"])

    def wait(b, k):
        return ("wait", b, k)

    def producer(kind, stages):
        for j in range(n_kv):
            s, use = j % stages, j // stages
            if use > 0:
                if release_barriers:
                    yield wait(f"e{kind}{s}", use - 1)
                elif kind == "k":
                    assert stages == SB
                    yield wait(f"sf{s}", use - 1)                                   # S of tile j-3 done
                else:
                    yield wait(f"or{(j - stages) % o_bars}", (j - stages) // o_bars)  # P.V of tile j-2 done
            pending.append((kind, j, s))
            yield ("nop",)

    def issue_s(j):
        yield wait(f"fk{j % K_STAGES}", j // K_STAGES)
        assert st["k"][j % K_STAGES] == j
        if j >= SB:
            if s_read_barrier:
                yield wait(f"sr{j % SB}", j // SB - 1)
            if not skip_pv_wait:
                yield wait(f"or{(j - SB) % o_bars}", (j - SB) // o_bars)   # P_{j-SB} in this S buffer consumed
                assert (j - SB) in st["pv"]
        q_s.append(("s", j))
        yield ("nop",)

    def pv(i):
        yield wait(f"pf{i % p_bars}", i // p_bars)
        assert st["P"][i] == N_SOFTMAX, "P.V issued before every warp wrote its part of P"
        yield wait(f"fv{i % V_STAGES}", i // V_STAGES)
        assert st["v"][i % V_STAGES] == i
        q_pv.append(("pv", i))
        yield ("nop",)

    def mma():
        yield wait("q", 0)
        for j in range(min(SB - 1, n_kv)):
            yield from issue_s(j)
        for j in range(n_kv):
            if j + SB - 1 < n_kv:
                yield from issue_s(j + SB - 1)
            yield from pv(j)

    def mma_s():
        yield wait("q", 0)
        for j in range(n_kv):
            yield from issue_s(j)

    def mma_pv():
        for i in range(n_kv):
            yield from pv(i)

    rescale = {j: rnd.random() < 0.3 for j in range(n_kv)}

    def softmax(w):
        q, half = w & 3, w // 4
        yield ("arrive", "q")
        for j in range(n_kv):
            yield wait(f"sf{j % SB}", j // SB)
            assert st["S"][j % SB] == j
            if s_read_barrier:
                yield ("arrive", f"sr{j % SB}", w)
            else:
                st["Sread"][j % SB].add(w)           # the read completes before this warp's P
                yield ("nop",)
            if row_split > 1:
                st["x"][q][j & 1][half] = j         # this part's maximum of tile j
                yield ("arrive", f"pair{q}{j & 1}")
                yield wait(f"pair{q}{j & 1}", j // 2)
                yield ("nop",)                       # the read may lag the wait
                assert st["x"][q][j & 1] == [j] * row_split, \
                    "a row maximum read before it was posted or after it was overwritten"
            if j >= 1 and rescale[j]:
                yield wait(f"or{(j - 1) % o_bars}", (j - 1) // o_bars)
                assert all(i in st["pv"] for i in range(j)), "O rescaled before every earlier P.V was done"
            if tail and j == n_kv - 1:
                if j >= V_STAGES:   # V_{j-2} (same stage) consumed, so landed: the wait below stays in window
                    yield wait(f"or{(j - V_STAGES) % o_bars}", (j - V_STAGES) // o_bars)
                yield wait(f"fv{j % V_STAGES}", j // V_STAGES)
                st["zeroed"].add((j, w))
            st["P"][j] += 1
            yield ("arrive", f"pf{j % p_bars}")
        if row_split > 1:
            yield ("arrive", f"pend{q}")
            yield wait(f"pend{q}", 0)
        yield wait(f"or{(n_kv - 1) % o_bars}", (n_kv - 1) // o_bars)
        assert all(i in st["pv"] for i in range(n_kv)), "O read before every P.V was done"

    mma_roles = {"mma_s": mma_s(), "mma_pv": mma_pv()} if issuers == 2 else {"mma": mma()}
    roles = {"pk": producer("k", K_STAGES), "pv": producer("v", V_STAGES), **mma_roles,
             **{f"w{w}": softmax(w) for w in range(N_SOFTMAX)}}
    cur = {k: None for k in roles}
    alive = set(roles)
    # each role runs at its own speed, so warps drift apart by many steps
    speed = {r: rnd.choice([1.0, 0.5, 0.1]) for r in roles}
    # in some runs the tile loads of one kind are slow to land
    slow = rnd.choice([None, "k", "v"])
    for _ in range(400000):
        heads = [q for q in mma_qs.values() if q]
        if not alive and not pending and not heads:
            return
        progressed = False
        op = None
        if (pending or heads) and rnd.random() < 0.4:
            k = rnd.randrange(len(pending) + len(heads))
            if k < len(pending) and pending[k][0] == slow and rnd.random() < 0.9:
                k = None                       # this load stays in flight a while longer
            if k is not None:
                op = pending.pop(k) if k < len(pending) else heads[k - len(pending)].pop(0)
        if op is not None:
            if op[0] == "k":
                st["k"][op[2]] = op[1]
                bars[f"fk{op[2]}"].arrive()
            elif op[0] == "v":
                st["v"][op[2]] = op[1]
                bars[f"fv{op[2]}"].arrive()
            elif op[0] == "s":
                j = op[1]
                prev = st["S"][j % SB]
                if prev is not None:
                    assert len(st["Sread"][j % SB]) == N_SOFTMAX, "S overwritten before all warps read it"
                    assert prev in st["pv"], "S overwritten while its P was still to be read by P.V"
                st["S"][j % SB] = j
                st["Sread"][j % SB] = set()
                bars[f"sf{j % SB}"].arrive()
                bars[f"ek{j % K_STAGES}"].arrive()
            else:
                i = op[1]
                if tail and i == n_kv - 1:
                    assert len([1 for (jj, _) in st["zeroed"] if jj == i]) == N_SOFTMAX, \
                        "P.V read the V tail before zeroing"
                assert all(k in st["pv"] for k in range(i)), "P.V completed out of order"
                st["pv"].add(i)
                bars[f"ev{i % V_STAGES}"].arrive()
                bars[f"or{i % o_bars}"].arrive()
            progressed = True
        order = list(alive)
        rnd.shuffle(order)
        for r in order:
            ev = cur[r]
            if rnd.random() > speed[r]:  # this role sits out the step
                if ev is None or ev[0] != "wait" or bars[ev[1]].done >= ev[2] + 1:
                    progressed = True    # (it could have moved)
                continue
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
                # a parity wait two phases ahead would pass at once
                assert b.done >= ev[2], f"{r} waits {ev[1]} phase {ev[2]} with only {b.done} phases done"
                if b.done >= ev[2] + 1:
                    cur[r] = None
                    progressed = True
            elif ev[0] == "arrive":
                bars[ev[1]].arrive()
                if ev[1].startswith("sr"):
                    st["Sread"][int(ev[1][2:])].add(ev[2])
                cur[r] = None
                progressed = True
            else:
                cur[r] = None
                progressed = True
        assert progressed or pending or any(mma_qs.values()), f"deadlock: {cur}"
    raise AssertionError("no termination")


@pytest.mark.parametrize("n_kv", [1, 2, 3, 4, 7])
@pytest.mark.parametrize("tail", [False, True])
def test_prefill_protocol(n_kv, tail):
    for seed in range(150):
        _prefill_run(n_kv, tail, seed)


@pytest.mark.parametrize("n_kv", [2, 7])
def test_prefill_protocol_with_stages_released_by_s_and_pv_barriers(n_kv):
    for seed in range(100):
        _prefill_run(n_kv, True, seed, release_barriers=False)


@pytest.mark.parametrize("n_kv", [1, 3, 7])
def test_prefill_protocol_with_two_mma_issuers(n_kv):
    # the same barriers with S and P.V issued by two threads, each chain
    # completing in its own order (a variant that measured slower on B200)
    for seed in range(100):
        _prefill_run(n_kv, True, seed, issuers=2)


@pytest.mark.parametrize("n_kv", [2, 5])
def test_prefill_protocol_with_rows_split_over_two_warps(n_kv):
    # the exchange of row maxima by tile parity, for a kernel that splits
    # each row over two warps of a lane quadrant
    for seed in range(100):
        _prefill_run(n_kv, True, seed, row_split=2)


@pytest.mark.parametrize("p_bars", [1, 2])
def test_prefill_protocol_catches_too_few_p_barriers(p_bars):
    # With fewer P barriers than S buffers, warps of another lane quadrant
    # that run ahead (their S is computed S_BUFS - 1 tiles early) can complete
    # a phase in place of a slow warp, and P.V would read that warp's columns
    # before its P is written. The model (warps at their own speeds) must find
    # that interleaving.
    failures = 0
    for seed in range(200):
        try:
            _prefill_run(5, False, seed, p_bars=p_bars)
        except AssertionError:
            failures += 1
    assert failures > 0


def test_prefill_protocol_catches_one_pv_barrier_for_all_buffers():
    # With three S buffers a warp can reach tile j before P.V of j-2 is done;
    # one P.V-done barrier for every tile then puts the rescale's wait for
    # P.V of j-1 two phases ahead, where a parity wait passes at once.
    failures = 0
    for seed in range(100):
        try:
            _prefill_run(5, False, seed, o_bars=1)
        except AssertionError:
            failures += 1
    assert failures > 0


def test_prefill_protocol_catches_s_reuse_without_the_pv_wait():
    # without the "S read" barrier the P.V-done wait is what keeps S_{j+3}
    # off a buffer still being read or holding P_j: dropping it must fail.
    # (With one issuer the model's in-order completion would hide the
    # mistake; the kernel does not rely on that order between different
    # MMAs, so the check runs with S and P.V on two issuers.)
    failures = 0
    for seed in range(100):
        try:
            _prefill_run(6, False, seed, skip_pv_wait=True, issuers=2)
        except AssertionError:
            failures += 1
    assert failures > 0

