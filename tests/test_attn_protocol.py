"""CPU model of the synchronisation inside the persistent attention kernel
(sparse_state_reuse_b200/csrc/attn_partial.cu), checked on random
interleavings.

The kernel's roles talk only through mbarriers in shared memory:
  * the producer warp takes each work item (from the work counter or a fixed
    stride), writes its index into a 2-slot ring in shared memory and
    publishes it (item_full); the MMA warp and the eight softmax warps read
    it and free the slot (item_empty); an index of -1 ends the CTA's work;
  * the producer warp arms a full barrier (arrive + expect_tx) and issues TMA
    loads of the Q tiles and of the two K and V stages;
  * the MMA warp issues tcgen05.mma (S = Q K^T into TMEM, O += P V with P
    read from the S columns) and tcgen05.commit arrivals;
  * eight softmax warps, four per 128-row Q tile, each own 32 TMEM lanes:
    they read S, write P in place, sometimes rescale O, and read O in the
    epilogue.
Each role below yields the same waits, arrivals and asynchronous operations
as the kernel, in the kernel's program order, with the kernel's own parity
expressions.  A scheduler interleaves them at random: a TMA load lands at
any later moment; MMAs complete in issue order at any later moment; a
commit arrives once every MMA issued before it has completed.

Checked on every interleaving:
  * progress: every wait ends (no interleaving stalls every role);
  * no phase aliasing: a parity wait can tell phase n from phase n + 1 only,
    so while a role waits for phase n its barrier never completes phase
    n + 1; and each parity the kernel computes is that of the phase it means;
  * no arrival beyond a barrier's count within one phase;
  * no data race on the item ring: the producer never writes a slot while
    a consumer reads it;
  * no data race on TMEM (S/P and O of each Q tile) or on the shared-memory
    tiles (Q0, Q1, K and V stages): a softmax access never overlaps an
    asynchronous operation in flight that writes the region (or reads it,
    when the access writes), and a load never overlaps an MMA that reads its
    region.  MMA after MMA is ordered by the tensor pipe and not checked;
  * at the end no operation is in flight and no barrier holds a half
    complete phase.
Planted mistakes (a dropped wait, an early release) must be caught, so that
a checker that passes everything would fail here.

The d = 64 and d = 96 kernels ("free S", fs=True below) keep P in TMEM
columns of its own and run one MMA warp per Q tile: each softmax warp
arrives on s_free once S is in its registers (the next Q K^T may then
overwrite S) and waits on p_free (the P V that read its previous P is done)
before it writes P again; each MMA warp follows its own tile, issuing the
next Q K^T after s_free and the P V after p_full; the Q, K and V stages and
the drain count one release per MMA warp, and for an item without a second
Q tile the second MMA warp only follows the stages and releases them.
"""
import random

import pytest

STAGES = 2
WARPS_PER_TILE = 4


class Violation(AssertionError):
    pass


class Bar:
    def __init__(self, name, count):
        self.name = name
        self.count = count
        self.pending = count
        self.tx = 0                    # loads armed but not landed
        self.phase = 0                 # phases completed

    def arrive(self):
        if self.pending == 0:
            raise Violation(f"arrival beyond the count of {self.name}")
        self.pending -= 1
        self._complete()

    def arm(self, loads):
        self.tx += loads
        self.arrive()

    def land(self):
        self.tx -= 1
        self._complete()

    def _complete(self):
        if self.pending == 0 and self.tx == 0:
            self.phase += 1
            self.pending = self.count


CONSUMERS = 1 + 2 * WARPS_PER_TILE      # the MMA warp and the eight softmax warps


def barriers(fs=False):
    releases = 2 if fs else 1                 # one per MMA warp
    b = {"q_full": 1, "q_empty": releases, "drain": releases}
    for s in range(2):
        b[f"item_full{s}"] = 1
        b[f"item_empty{s}"] = CONSUMERS + (1 if fs else 0)
    for s in range(STAGES):
        b[f"k_full{s}"] = b[f"v_full{s}"] = 1
        b[f"k_empty{s}"] = b[f"v_empty{s}"] = releases
    for k in range(2):
        b[f"s_full{k}"] = 1
        b[f"p_full{k}"] = WARPS_PER_TILE      # one arrival per softmax warp
        b[f"o_full{k}"] = 1
        b[f"o_empty{k}"] = WARPS_PER_TILE
        if fs:
            b[f"s_free{k}"] = WARPS_PER_TILE
            b[f"p_free{k}"] = 1
    return {n: Bar(n, c) for n, c in b.items()}


# ---------------------------------------------------------------- the roles
# An item is one (query partition, batch-head, pair of Q tiles) of a CTA:
# (has1, [key tiles of each fresh unit of the partition]).
#
# A wait is ("wait", barrier, parity, phase index[, abortable]); the role gets
# back True when the phase completed, False when it gave up (its time limit
# ran out, or another role set the CTA's abort flag), as the kernel's bounded
# waits return.  Waits that are not abortable are the drains of the stop
# path, which wait for work already issued and ignore the abort flag.

def W(bar, parity, n, abortable=True):
    return ("wait", bar, parity, n, abortable)


def publish(ic, mut):
    """The producer writes item ic's index (or the end marker) into slot
    ic % 2 once every consumer has read the slot's previous entry."""
    s = ic & 1
    if mut != "producer_skips_item_empty":
        ok = yield W(f"item_empty{s}", ((ic >> 1) & 1) ^ 1, (ic >> 1) - 1)
        if not ok:
            return False
    yield ("hold", f"ITEM{s}", "w")
    yield ("release", f"ITEM{s}")
    yield ("arrive", f"item_full{s}")
    return True


def take(ic, mut):
    """A consumer reads entry ic of the ring and frees the slot."""
    s = ic & 1
    ok = yield W(f"item_full{s}", (ic >> 1) & 1, ic >> 1)
    if not ok:
        return False
    if mut == "consumer_frees_slot_before_reading":
        yield ("arrive", f"item_empty{s}")
    yield ("hold", f"ITEM{s}", "r")
    yield ("release", f"ITEM{s}")
    if mut != "consumer_frees_slot_before_reading":
        yield ("arrive", f"item_empty{s}")
    return True


def producer(items, mut):
    kc = vc = uc = 0
    q_armed = None              # phase index of the last arming, per barrier
    k_armed, v_armed = {}, {}
    ok = True
    ic = 0
    for has1, Ts in items:
        ok = yield from publish(ic, mut)
        ic += 1
        if not ok:
            break
        ok = yield W("q_empty", (uc & 1) ^ 1, uc - 1)
        if not ok:
            break
        yield ("arm", "q_full", 2 if has1 else 1)
        q_armed = uc
        yield ("load", "Q0", "q_full")
        if has1:
            yield ("load", "Q1", "q_full")
        for T in Ts:
            for _ in range(T):
                s = kc % STAGES
                if mut != "producer_skips_k_empty":
                    ok = yield W(f"k_empty{s}", ((kc // STAGES) & 1) ^ 1, kc // STAGES - 1)
                    if not ok:
                        break
                yield ("arm", f"k_full{s}", 1)
                k_armed[s] = kc // STAGES
                yield ("load", f"K{s}", f"k_full{s}")
                kc += 1
                s = vc % STAGES
                ok = yield W(f"v_empty{s}", ((vc // STAGES) & 1) ^ 1, vc // STAGES - 1)
                if not ok:
                    break
                yield ("arm", f"v_full{s}", 1)
                v_armed[s] = vc // STAGES
                yield ("load", f"V{s}", f"v_full{s}")
                vc += 1
            if not ok:
                break
        if not ok:
            break
        uc += 1
    if ok:
        ok = yield from publish(ic, mut)          # the end marker
    # every load issued lands before the warp exits, on both paths: when
    # another role gave up, this warp may still end its loop with ok (each
    # of its last waits completed at once) while nothing consumes its loads
    drain = mut != "producer_stops_without_drain"
    if mut == "producer_drains_only_after_giving_up":
        drain = not ok
    if drain:
        if q_armed is not None:
            yield W("q_full", q_armed & 1, q_armed, False)
        for s in range(STAGES):
            if s in k_armed:
                yield W(f"k_full{s}", k_armed[s] & 1, k_armed[s], False)
            if s in v_armed:
                yield W(f"v_full{s}", v_armed[s] & 1, v_armed[s], False)


def mma(items, mut):
    kc = vc = uc = 0
    pc = [0, 0]
    oc = [0, 0]
    ok = True

    def qk(k, ks):
        return ("mma", {f"Q{k}", f"K{ks}"}, {f"S{k}"})

    def pv(k, vs, acc):
        return ("mma", {f"S{k}", f"V{vs}"} | ({f"O{k}"} if acc else set()), {f"O{k}"})

    ic = 0
    for has1, Ts in items:
        ok = yield from take(ic, mut)
        ic += 1
        if not ok:
            break
        ok = yield W("q_full", uc & 1, uc)
        if not ok:
            break
        for fi, T in enumerate(Ts):
            last_pair = fi + 1 == len(Ts)
            ks = kc % STAGES
            ok = yield W(f"k_full{ks}", (kc // STAGES) & 1, kc // STAGES)
            if not ok:
                break
            if mut == "k_released_before_qk":
                yield ("commit", f"k_empty{ks}")
            yield qk(0, ks)
            yield ("commit", "s_full0")
            if has1:
                yield qk(1, ks)
                yield ("commit", "s_full1")
            if mut != "k_released_before_qk":
                yield ("commit", f"k_empty{ks}")
            kc += 1
            if T == 1 and last_pair:
                yield ("commit", "q_empty")
            for t in range(T):
                vs = vc % STAGES
                ok = yield W(f"v_full{vs}", (vc // STAGES) & 1, vc // STAGES)
                if not ok:
                    break
                more = t + 1 < T
                for k in range(2):
                    if k == 1 and not has1:
                        break
                    if not (mut == "mma_skips_p_full" and k == 0):
                        ok = yield W(f"p_full{k}", pc[k] & 1, pc[k])
                        if not ok:
                            break
                    pc[k] += 1
                    if t == 0:
                        if mut != "mma_skips_o_empty":
                            ok = yield W(f"o_empty{k}", (oc[k] & 1) ^ 1, oc[k] - 1)
                            if not ok:
                                break
                        oc[k] += 1
                    yield pv(k, vs, t > 0)
                    if not more:
                        yield ("commit", f"o_full{k}")
                    if more:
                        ks2 = kc % STAGES
                        if k == 0:
                            ok = yield W(f"k_full{ks2}", (kc // STAGES) & 1, kc // STAGES)
                            if not ok:
                                break
                        yield qk(k, ks2)
                        yield ("commit", f"s_full{k}")
                if not ok:
                    break
                yield ("commit", f"v_empty{vs}")
                vc += 1
                if more:
                    yield ("commit", f"k_empty{kc % STAGES}")
                    kc += 1
                    if t + 2 == T and last_pair:
                        yield ("commit", "q_empty")
            if not ok:
                break
        if not ok:
            break
        uc += 1
    if ok:
        yield from take(ic, mut)                  # the end marker
    # drain: every MMA issued must finish before TMEM is released
    if mut != "mma_stops_without_drain":
        yield ("commit", "drain")
        yield W("drain", 0, 0, False)


def softmax_warp(k, items, rng, rescale_p, mut):
    sc = ofc = 0
    S, O = f"S{k}", f"O{k}"
    ok = True
    ic = 0
    for has1, Ts in items:
        ok = yield from take(ic, mut)
        ic += 1
        if not ok:
            break
        if k == 1 and not has1:
            continue
        for T in Ts:
            for t in range(T):
                ok = yield W(f"s_full{k}", sc & 1, sc)
                if not ok:
                    break
                sc += 1
                yield ("hold", S, "w")                 # read S, write P over it
                if t > 0 and rng.random() < rescale_p:
                    yield ("hold", O, "w")             # O *= alpha
                    yield ("release", O)
                if mut == "p_full_before_p_written":
                    yield ("arrive", f"p_full{k}")
                    yield ("release", S)
                else:
                    yield ("release", S)
                    yield ("arrive", f"p_full{k}")
            if not ok:
                break
            if mut != "softmax_skips_o_full":
                ok = yield W(f"o_full{k}", ofc & 1, ofc)
                if not ok:
                    break
            ofc += 1
            yield ("hold", O, "r")                     # O into registers
            yield ("release", O)
            yield ("arrive", f"o_empty{k}")
        if not ok:
            break
    if ok:
        yield from take(ic, mut)                  # the end marker


def mma_fs(k, items, mut):
    """MMA warp 9 + k of the free-S kernels: Q tile k only."""
    kc = vc = uc = 0
    pc = oc = sf = 0
    ok = True

    def qk(ks):
        return ("mma", {f"Q{k}", f"K{ks}"}, {f"S{k}"})

    def pv(vs, acc):
        return ("mma", {f"P{k}", f"V{vs}"} | ({f"O{k}"} if acc else set()), {f"O{k}"})

    ic = 0
    for has1, Ts in items:
        ok = yield from take(ic, mut)
        ic += 1
        if not ok:
            break
        n_steps = sum(Ts)
        ok = yield W("q_full", uc & 1, uc)
        if not ok:
            break
        uc += 1
        if k == 1 and not has1:
            # no second Q tile: follow the stages and release them
            yield ("commit", "q_empty")
            for _ in range(n_steps):
                ok = yield W(f"k_full{kc % STAGES}", (kc // STAGES) & 1, kc // STAGES)
                if not ok:
                    break
                if mut != "fs_idle_warp_skips_release":
                    yield ("commit", f"k_empty{kc % STAGES}")
                kc += 1
                ok = yield W(f"v_full{vc % STAGES}", (vc // STAGES) & 1, vc // STAGES)
                if not ok:
                    break
                yield ("commit", f"v_empty{vc % STAGES}")
                vc += 1
            if not ok:
                break
            continue
        ok = yield W(f"k_full{kc % STAGES}", (kc // STAGES) & 1, kc // STAGES)
        if not ok:
            break
        yield qk(kc % STAGES)
        yield ("commit", f"s_full{k}")
        yield ("commit", f"k_empty{kc % STAGES}")
        kc += 1
        if n_steps == 1:
            yield ("commit", "q_empty")
        f, t, T = 0, 0, Ts[0]
        for n in range(n_steps):
            if mut != "fs_mma_skips_s_free":
                ok = yield W(f"s_free{k}", sf & 1, sf)
                if not ok:
                    break
            sf += 1
            if n + 1 < n_steps:
                ok = yield W(f"k_full{kc % STAGES}", (kc // STAGES) & 1, kc // STAGES)
                if not ok:
                    break
                yield qk(kc % STAGES)
                yield ("commit", f"s_full{k}")
                yield ("commit", f"k_empty{kc % STAGES}")
                kc += 1
                if n + 2 == n_steps:
                    yield ("commit", "q_empty")
            ok = yield W(f"v_full{vc % STAGES}", (vc // STAGES) & 1, vc // STAGES)
            if not ok:
                break
            ok = yield W(f"p_full{k}", pc & 1, pc)
            if not ok:
                break
            pc += 1
            if t == 0:
                ok = yield W(f"o_empty{k}", (oc & 1) ^ 1, oc - 1)
                if not ok:
                    break
                oc += 1
            yield pv(vc % STAGES, t > 0)
            yield ("commit", f"p_free{k}")
            yield ("commit", f"v_empty{vc % STAGES}")
            vc += 1
            if t + 1 == T:
                yield ("commit", f"o_full{k}")
                t, f = 0, f + 1
                if f < len(Ts):
                    T = Ts[f]
            else:
                t += 1
        if not ok:
            break
    if ok:
        yield from take(ic, mut)                  # the end marker
    yield ("commit", "drain")
    yield W("drain", 0, 0, False)


def softmax_warp_fs(k, items, rng, rescale_p, mut):
    sc = ofc = pst = 0
    S, P, O = f"S{k}", f"P{k}", f"O{k}"
    ok = True
    ic = 0
    for has1, Ts in items:
        ok = yield from take(ic, mut)
        ic += 1
        if not ok:
            break
        if k == 1 and not has1:
            continue
        for T in Ts:
            for t in range(T):
                ok = yield W(f"s_full{k}", sc & 1, sc)
                if not ok:
                    break
                sc += 1
                if mut == "fs_s_free_before_s_read":
                    yield ("arrive", f"s_free{k}")
                yield ("hold", S, "r")                 # S into registers
                yield ("release", S)
                if mut != "fs_s_free_before_s_read":
                    yield ("arrive", f"s_free{k}")
                pv_done = pst == 0 or mut == "fs_softmax_skips_p_free"
                if t > 0 and rng.random() < rescale_p:
                    if not pv_done:
                        ok = yield W(f"p_free{k}", (pst - 1) & 1, pst - 1)
                        if not ok:
                            break
                        pv_done = True
                    yield ("hold", O, "w")             # O *= alpha
                    yield ("release", O)
                # the P row is formed in registers (no TMEM access) before
                # this wait; only its store touches P_k
                if not pv_done:
                    ok = yield W(f"p_free{k}", (pst - 1) & 1, pst - 1)
                    if not ok:
                        break
                yield ("hold", P, "w")                 # the probabilities of this tile
                yield ("release", P)
                yield ("arrive", f"p_full{k}")
                pst += 1
            if not ok:
                break
            ok = yield W(f"o_full{k}", ofc & 1, ofc)
            if not ok:
                break
            ofc += 1
            yield ("hold", O, "r")
            yield ("release", O)
            yield ("arrive", f"o_empty{k}")
        if not ok:
            break
    if ok:
        yield from take(ic, mut)                  # the end marker


# ---------------------------------------------------------------- scheduler

def conflicts(reads_a, writes_a, reads_b, writes_b):
    return bool(writes_a & (reads_b | writes_b)) or bool(reads_a & writes_b)


def run(items, seed, rescale_p=0.5, mut=None, timeout_p=0.0, max_steps=2_000_000, fs=False):
    """Interleave the roles at random; raise Violation on any broken rule.

    timeout_p: per scheduling step, the chance that one role blocked on an
    abortable wait runs out of time (which sets the abort flag; from then on
    every role blocked on an abortable wait may give up).  Returns the
    barriers and whether the run aborted."""
    rng = random.Random(seed)
    B = barriers(fs)
    roles = {"producer": producer(items, mut)}
    if fs:
        roles["mma0"], roles["mma1"] = mma_fs(0, items, mut), mma_fs(1, items, mut)
    else:
        roles["mma"] = mma(items, mut)
    sm = softmax_warp_fs if fs else softmax_warp
    for k in range(2):
        for w in range(WARPS_PER_TILE):
            roles[f"softmax{k}.{w}"] = sm(k, items, random.Random(rng.random()), rescale_p, mut)
    nxt = {r: next(g, None) for r, g in roles.items()}
    loads = []                 # in flight: (region, barrier)
    # in issue order, tagged with the issuing role: ("mma", reads, writes) |
    # ("commit", barrier).  Each role's operations complete in its issue
    # order, those of different MMA warps in any order between them; a
    # commit arrives once every MMA its own role issued before it is done.
    mma_q = []
    holds = {}                 # role -> {region: mode}
    aborted = False

    def check_wait(role, op):
        _, name, parity, n, _ = op
        if parity != (n & 1):
            raise Violation(f"{role}: parity {parity} for phase {n} of {name}")
        if B[name].phase > n + 1:
            raise Violation(f"{role}: {name} completed phase {n + 1} while it waits for phase {n}")

    def mma_in_flight():
        return [op for _, op in mma_q if op[0] == "mma"]

    def advance(role, value=None):
        try:
            nxt[role] = roles[role].send(value)
        except StopIteration:
            nxt[role] = None
        if all(op is None for op in nxt.values()):
            # the CTA exits (TMEM is freed): nothing of it may still be in flight
            if mma_q:
                raise Violation("MMAs in flight when the CTA exits")
            if loads:
                raise Violation("loads in flight when the CTA exits")

    for _ in range(max_steps):
        choices = []
        blocked = []
        for r, op in nxt.items():
            if op is None:
                continue
            if op[0] == "wait":
                check_wait(r, op)
                if B[op[1]].phase >= op[3] + 1:
                    choices.append(("role", r))
                elif op[4]:
                    blocked.append(r)
                    if aborted:
                        choices.append(("give_up", r))
            else:
                choices.append(("role", r))
        if blocked and not aborted and timeout_p and rng.random() < timeout_p:
            choices = [("give_up", rng.choice(blocked))]
        if mma_q:
            choices.append(("mma", None))
        choices.extend(("land", i) for i in range(len(loads)))
        if not choices:
            if all(op is None for op in nxt.values()):
                break
            waiting = {r: op for r, op in nxt.items() if op is not None}
            raise Violation(f"no role can proceed: {waiting}")
        kind, x = rng.choice(choices)
        if kind == "mma":
            issuers = sorted({r for r, _ in mma_q})
            issuer = issuers[0] if len(issuers) == 1 else rng.choice(issuers)
            i = next(j for j, (r, _) in enumerate(mma_q) if r == issuer)
            _, op = mma_q.pop(i)
            if op[0] == "commit":
                B[op[1]].arrive()
            continue
        if kind == "land":
            region, name = loads.pop(x)
            B[name].land()
            continue
        if kind == "give_up":
            aborted = True
            advance(x, False)
            continue
        role, op = x, nxt[x]
        what = op[0]
        if what == "arrive":
            B[op[1]].arrive()
        elif what == "arm":
            B[op[1]].arm(op[2])
        elif what == "load":
            region = op[1]
            for m in mma_in_flight():
                if conflicts(set(), {region}, m[1], m[2]):
                    raise Violation(f"load of {region} while an MMA on it is in flight")
            if any(r == region for r, _ in loads):
                raise Violation(f"two loads of {region} in flight")
            for h in holds.values():
                if region in h:
                    raise Violation(f"load of {region} while a softmax warp holds it")
            loads.append((region, op[2]))
        elif what == "mma":
            _, reads, writes = op
            for region, _ in loads:
                if region in reads | writes:
                    raise Violation(f"MMA on {region} before its load landed")
            for h in holds.values():
                for region, mode in h.items():
                    if conflicts(reads, writes, {region} if mode == "r" else set(),
                                 {region} if mode == "w" else set()):
                        raise Violation(f"MMA on {region} while a softmax warp holds it ({mode})")
            mma_q.append((role, op))
        elif what == "commit":
            mma_q.append((role, op))
        elif what == "hold":
            region, mode = op[1], op[2]
            if region.startswith("ITEM"):
                # the ring slots are plain shared memory written and read by roles
                for other, h in holds.items():
                    if other != role and region in h and "w" in (mode, h[region]):
                        raise Violation(f"{role} and {other} race on {region}")
            r_set = {region}
            w_set = {region} if mode == "w" else set()
            for m in mma_in_flight():
                if conflicts(r_set, w_set, m[1], m[2]):
                    raise Violation(f"{role} touches {region} ({mode}) under an MMA in flight")
            holds.setdefault(role, {})[region] = mode
        elif what == "release":
            del holds[role][op[1]]
        advance(role, True if what == "wait" else None)
    else:
        raise Violation("step limit reached")
    if any(holds.values()):
        raise Violation("a region is still held at the end")
    if not aborted:
        for b in B.values():
            if b.pending != b.count or b.tx != 0:
                raise Violation(f"{b.name} ends inside a phase")
    return B, aborted


def random_items(rng):
    items = []
    for _ in range(rng.randint(1, 5)):
        has1 = rng.random() < 0.7
        items.append((has1, [rng.choice([1, 1, 2, 3, 5]) for _ in range(rng.randint(1, 4))]))
    return items


@pytest.mark.parametrize("seed", range(60))
def test_protocol_on_random_items_and_interleavings(seed):
    rng = random.Random(1000 + seed)
    items = random_items(rng)
    B, aborted = run(items, seed, rescale_p=rng.choice([0.0, 0.3, 1.0]))
    assert not aborted
    # every barrier completed exactly the phases its traffic implies
    n_units = sum(len(Ts) for _, Ts in items)
    n_tiles = sum(sum(Ts) for _, Ts in items)
    n_units1 = sum(len(Ts) for has1, Ts in items if has1)
    n_tiles1 = sum(sum(Ts) for has1, Ts in items if has1)
    assert B["q_full"].phase == B["q_empty"].phase == len(items)
    # every item and the end marker went through the ring
    assert B["item_full0"].phase + B["item_full1"].phase == len(items) + 1
    assert B["item_empty0"].phase + B["item_empty1"].phase == len(items) + 1
    assert sum(B[f"k_full{s}"].phase for s in range(STAGES)) == n_tiles
    assert sum(B[f"v_empty{s}"].phase for s in range(STAGES)) == n_tiles
    assert B["s_full0"].phase == B["p_full0"].phase == n_tiles
    assert B["s_full1"].phase == B["p_full1"].phase == n_tiles1
    assert B["o_full0"].phase == B["o_empty0"].phase == n_units
    assert B["o_full1"].phase == B["o_empty1"].phase == n_units1
    assert B["drain"].phase == 1


@pytest.mark.parametrize("items", [
    [(False, [1])],                       # one tile, one Q tile
    [(True, [1])],
    [(True, [1] * 7)],                    # many one-tile units: q_empty on the first QK
    [(False, [2]), (True, [1]), (False, [3, 1])],
    [(True, [9])],                        # a long unit: both stages cycle many times
], ids=["T1_tile0", "T1_both", "units_of_one_tile", "mixed", "long_unit"])
def test_protocol_edge_items(items):
    for seed in range(20):
        run(items, seed)


@pytest.mark.parametrize("mut", ["mma_skips_p_full", "softmax_skips_o_full", "k_released_before_qk",
                                 "p_full_before_p_written", "producer_skips_k_empty",
                                 "producer_skips_item_empty", "consumer_frees_slot_before_reading"])
def test_planted_mistakes_are_caught(mut):
    # items without a second Q tile let the MMA warp and the producer run
    # ahead of the second softmax warpgroup, which only reads their entries
    item_lists = [[(True, [3, 2]), (True, [1, 4]), (False, [2])],
                  [(True, [3]), (False, [1]), (False, [1]), (False, [1]), (True, [1])]]
    caught = 0
    for items in item_lists:
        for seed in range(40):
            try:
                run(items, seed, mut=mut)
            except Violation:
                caught += 1
    assert caught > 0, mut


def test_o_empty_wait_is_implied_by_p_full():
    """The MMA warp's o_empty wait before the first P V of a unit never
    blocks: each softmax warp arrives on o_empty before it reaches the next
    unit's first tile, and that P V already waits for all four warps' p_full
    arrivals.  The wait stays in the kernel as a guard; the model shows it is
    not what orders the epilogue's O reads before the next unit's P V."""
    items = [(True, [3, 2]), (True, [1, 4]), (False, [2])]
    for seed in range(40):
        run(items, seed, mut="mma_skips_o_empty")


@pytest.mark.parametrize("seed", range(40))
def test_stop_path_after_a_timeout(seed):
    """A wait that runs out of time sets the CTA's abort flag; every role then
    leaves at its next wait that has not completed.  The stop path must end
    (its drains wait only for work already issued) and leave no TMA load or
    MMA in flight when the CTA exits and frees its TMEM.  A producer that
    drained only after giving up itself fails this (its last loads can be
    in flight when the CTA exits after the MMA warp gave up)."""
    rng = random.Random(5000 + seed)
    items = random_items(rng)
    aborted_runs = 0
    for timeout_p in (0.002, 0.02, 0.2):
        _, aborted = run(items, seed, timeout_p=timeout_p)
        aborted_runs += aborted
    assert aborted_runs > 0


@pytest.mark.parametrize("mut", ["producer_stops_without_drain",
                                 "producer_drains_only_after_giving_up",
                                 "mma_stops_without_drain"])
def test_stop_path_without_its_drain_is_caught(mut):
    caught = 0
    for items in ([(True, [2])], [(True, [3, 2]), (True, [1, 4]), (False, [2])]):
        for seed in range(60):
            try:
                run(items, seed, mut=mut, timeout_p=0.05)
            except Violation:
                caught += 1
    assert caught > 0, mut


def cta_items(part_off, fresh_rows, BH, cta, grid, BM=128, BN=128):
    """The item list one CTA of the persistent grid walks without a work
    counter: items are (partition, batch-head, pair of 128-row Q tiles) in
    the kernel's order -- b*h-major, every partition's last pair of Q tiles
    after all the others -- taken with stride `grid`; fresh_rows[i] lists
    the key counts of the fresh units of partition i."""
    P = len(part_off) - 1
    Lmax = max(part_off[i + 1] - part_off[i] for i in range(P))
    nqt2 = -(-Lmax // (2 * BM))
    n_main = P * BH * (nqt2 - 1)
    items = []
    for it in range(cta, P * BH * nqt2, grid):
        if it < n_main:
            qt2, rest = it % (nqt2 - 1), it // (nqt2 - 1)
        else:
            qt2, rest = nqt2 - 1, it - n_main
        i = rest % P
        rem = part_off[i + 1] - part_off[i] - qt2 * 2 * BM
        if rem <= 0 or not fresh_rows[i]:
            continue                     # not live: no role touches it
        items.append((rem > BM, [-(-Lk // BN) for Lk in fresh_rows[i]]))
    return items


@pytest.mark.parametrize("cta", [0, 147])
def test_protocol_on_a_frame_tile_cta(cta):
    """One CTA of the 148-CTA grid on 8 frames of 3600 tokens, 24 heads, every
    active pair fresh: about 20 items of 2 to 4 units of 29 key tiles, the
    last Q-tile pair of each partition with a single tile of 16 rows."""
    F, L = 8, 3600
    part_off = [f * L for f in range(F + 1)]
    fresh_rows = [[L] * len({0, f - 1, f, f + 1} & set(range(F))) for f in range(F)]
    items = cta_items(part_off, fresh_rows, 24, cta, 148)
    assert 15 <= len(items) <= 25 and any(not has1 for has1, _ in items)
    assert {T for _, Ts in items for T in Ts} == {29}
    for seed in range(2):
        B, aborted = run(items, seed, rescale_p=0.05)
        assert not aborted
        assert B["o_full0"].phase == sum(len(Ts) for _, Ts in items)


# ------------------------------------------------ free S (d = 64 and 96)

@pytest.mark.parametrize("seed", range(60))
def test_free_s_protocol_on_random_items_and_interleavings(seed):
    rng = random.Random(3000 + seed)
    items = random_items(rng)
    B, aborted = run(items, seed, rescale_p=rng.choice([0.0, 0.3, 1.0]), fs=True)
    assert not aborted
    n_units = sum(len(Ts) for _, Ts in items)
    n_tiles = sum(sum(Ts) for _, Ts in items)
    n_units1 = sum(len(Ts) for has1, Ts in items if has1)
    n_tiles1 = sum(sum(Ts) for has1, Ts in items if has1)
    assert B["q_full"].phase == B["q_empty"].phase == len(items)
    assert B["item_empty0"].phase + B["item_empty1"].phase == len(items) + 1
    assert sum(B[f"k_empty{s}"].phase for s in range(STAGES)) == n_tiles
    assert sum(B[f"v_empty{s}"].phase for s in range(STAGES)) == n_tiles
    for k, (tiles, units) in enumerate(((n_tiles, n_units), (n_tiles1, n_units1))):
        assert B[f"s_full{k}"].phase == B[f"s_free{k}"].phase == tiles
        assert B[f"p_full{k}"].phase == B[f"p_free{k}"].phase == tiles
        assert B[f"o_full{k}"].phase == B[f"o_empty{k}"].phase == units
    assert B["drain"].phase == 1


@pytest.mark.parametrize("items", [
    [(False, [1])],
    [(True, [1])],
    [(True, [1] * 7)],
    [(False, [2]), (True, [1]), (False, [3, 1])],
    [(True, [9])],
    [(False, [4]), (False, [1]), (True, [2, 2])],   # the second MMA warp follows two items idle
], ids=["T1_tile0", "T1_both", "units_of_one_tile", "mixed", "long_unit", "idle_items"])
def test_free_s_protocol_edge_items(items):
    for seed in range(20):
        run(items, seed, fs=True)


@pytest.mark.parametrize("mut", ["fs_s_free_before_s_read", "fs_softmax_skips_p_free",
                                 "fs_mma_skips_s_free", "fs_idle_warp_skips_release"])
def test_free_s_planted_mistakes_are_caught(mut):
    item_lists = [[(True, [3, 2]), (True, [1, 4]), (False, [2])],
                  [(True, [3]), (False, [1]), (False, [1]), (True, [2])]]
    caught = 0
    for items in item_lists:
        for seed in range(40):
            try:
                run(items, seed, mut=mut, fs=True)
            except Violation:
                caught += 1
    assert caught > 0, mut


@pytest.mark.parametrize("seed", range(20))
def test_free_s_stop_path_after_a_timeout(seed):
    rng = random.Random(7000 + seed)
    items = random_items(rng)
    aborted_runs = 0
    for timeout_p in (0.002, 0.02, 0.2):
        _, aborted = run(items, seed, timeout_p=timeout_p, fs=True)
        aborted_runs += aborted
    assert aborted_runs > 0


@pytest.mark.parametrize("cta", [0, 147])
def test_free_s_protocol_on_a_frame_tile_cta(cta):
    """The d = 96 kernel on 8 frames of 3600 tokens: 96-key tiles, 38 per
    unit (the last one 48 keys)."""
    F, L = 8, 3600
    part_off = [f * L for f in range(F + 1)]
    fresh_rows = [[L] * len({0, f - 1, f, f + 1} & set(range(F))) for f in range(F)]
    items = cta_items(part_off, fresh_rows, 24, cta, 148, BN=96)
    assert {T for _, Ts in items for T in Ts} == {38}
    B, aborted = run(items, cta, rescale_p=0.05, fs=True)
    assert not aborted
    assert B["p_free0"].phase == sum(sum(Ts) for _, Ts in items)
