"""Host-side model of the attention kernel's mbarrier protocol (one CTA).

attn_kernel hands work between its warp roles only through mbarriers. This
model runs the same roles as Python generators -- the list scheduler (warp 2),
the K and V producer lanes (warp 0), the S issuer (warp 1), the two PV issuers
(warps 3 and 12) and the eight softmax warps (two warpgroups) -- with each
barrier's arrival count and each wait's phase parity as in the kernel. TMA
copies and MMA commits complete later, in issue order per issuing thread, at
times the scheduler of the model picks. A run reports "ok", a deadlock (no
role can move), or raises Hazard when a role reads or overwrites a buffer
(Q, K stage, V stage, S buffer, P, O) out of turn, tracked by block numbers.

mbarrier semantics: a barrier completes a phase when its pending count reaches
zero; a wait on parity p returns once the phase with parity p has completed,
that is, while the current phase's parity differs from p. A waiter that falls
two phases behind therefore waits for good: that is the aliasing the model
looks for.

Items are given as their key-block counts. `slot_readers_release` (the
kernel's counts) has the list-slot barrier count every role that reads the
slot (13 arrivals); False models the earlier kernel, whose barrier counted the
eight softmax warps alone. `faults` plants protocol mistakes (the tests check
that the model catches them): "s_skips_pv_done" (the S issuer reuses an S
buffer without waiting for the PVs that read its P) and "softmax_parity" (the
softmax waits on the wrong phase parity), "mma_no_drain" and "tma_no_drain"
(the MMA issuers or the producer lanes leave without draining).

Bounded waits and the abort path: every wait of the kernel gives up after a
time limit. When no role can move and nothing is in flight, the model lets one
waiting role run out of time: it raises the abort flag. From then on a wait
whose phase has not completed returns false and the role leaves its loop (a
wait whose phase has completed still returns true, as try_wait does). On the
way out the producer lanes wait for their own copies in flight, and each MMA
issuer commits to the drain barrier (counted by the three issuers) and waits
for it, so that no copy or MMA is in flight when the CTA ends and frees its
tensor memory; the model raises Hazard otherwise. `hold` models the kernel's
test hold: the softmax warps wait, at their first block, on a barrier nothing
arrives on. `timeout_p` lets a wait that has not passed run out early, with
probability timeout_p per step, while copies and MMAs are still in flight (a
limit shorter than a copy's latency, as a caller may set one).
"""
from __future__ import annotations

import random

K_STAGES, V_STAGES, S_BUFS = 2, 3, 2


class Hazard(Exception):
    pass


class Bar:
    def __init__(self, count):
        self.count, self.pending, self.phase = count, count, 0

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0
        if self.pending == 0:
            self.phase += 1
            self.pending = self.count

    def passed(self, parity):
        return (self.phase & 1) != parity


def _check(cond, msg):
    if not cond:
        raise Hazard(msg)


def run(blocks_per_item, rng, slot_readers_release=True, starve=(), faults=(), hold=False, timeout_p=0.0,
        max_steps=1_000_000):
    n_items = len(blocks_per_item)
    bars = {"QFULL": Bar(1), "QEMPTY": Bar(1), "OFULL": Bar(2), "OFREE": Bar(8), "LX": Bar(8),
            "HOLD": Bar(1), "DRAIN": Bar(3)}
    for i in range(K_STAGES):
        bars[f"KFULL{i}"], bars[f"KEMPTY{i}"] = Bar(1), Bar(1)
    for i in range(V_STAGES):
        bars[f"VFULL{i}"], bars[f"VEMPTY{i}"] = Bar(1), Bar(2)      # both PV issuers release a V stage
    for i in range(S_BUFS):
        bars[f"SFULL{i}"], bars[f"PDONE{i}"] = Bar(1), Bar(2)     # PDONE: both PV issuers' MMAs of the buffer
        for w in range(2):
            bars[f"PFULL{w}_{i}"] = Bar(4)
    for i in range(2):
        bars[f"LFULL{i}"] = Bar(32)
        bars[f"LEMPTY{i}"] = Bar(13 if slot_readers_release else 8)
    st = {"info": [None, None], "Q": None, "q_free": -1, "K": [None] * K_STAGES, "V": [None] * V_STAGES,
          "S": [None] * S_BUFS, "s_done": -1, "pv_done": [-1, -1], "epilogue_done": -1, "epi": {}}
    pending = []   # (issuer, completion)
    flags = {"abort": False}

    def later(issuer, fn):
        pending.append((issuer, fn))

    def wait(name, parity):
        return name, parity

    def drain_copies(issuer):       # a producer lane waits for its own copies in flight
        return "copies", issuer

    def drain_mmas(issuer):         # an MMA issuer: commit to DRAIN, then wait for all three commits
        later(issuer, lambda: bars["DRAIN"].arrive())
        return "drain", 0

    def scheduler():
        for it in range(n_items + 1):
            slot = it & 1
            if not (yield wait(f"LEMPTY{slot}", ((it >> 1) & 1) ^ 1)):
                return
            st["info"][slot] = (it, blocks_per_item[it]) if it < n_items else None
            for _ in range(32):
                bars[f"LFULL{slot}"].arrive()
            if it == n_items:
                return

    def producer(is_k):
        g, stage, ph = 0, 0, 0
        n_st = K_STAGES if is_k else V_STAGES
        ok = True
        for it in range(n_items + 1):
            slot = it & 1
            if not (ok := (yield wait(f"LFULL{slot}", (it >> 1) & 1))):
                break
            info = st["info"][slot]
            if info is None:
                break
            _check(info[0] == it, f"{'K' if is_k else 'V'} producer took item {info[0]} for {it}")
            if is_k:
                if not (ok := (yield wait("QEMPTY", (it & 1) ^ 1))):
                    break
                _check(st["q_free"] >= it - 1, "Q reloaded while in use")
                later("tmaK", lambda it=it: (st.__setitem__("Q", it), bars["QFULL"].arrive()))
            for _ in range(info[1]):
                if not (ok := (yield wait(f"{'K' if is_k else 'V'}EMPTY{stage}", ph ^ 1))):
                    break
                consumed = st["s_done"] if is_k else min(st["pv_done"])
                _check(consumed >= g - n_st, f"stage {stage} reloaded before block {g - n_st} was used")

                def land(stage=stage, g=g):
                    (st["K"] if is_k else st["V"])[stage] = g
                    bars[f"{'K' if is_k else 'V'}FULL{stage}"].arrive()
                later("tmaK" if is_k else "tmaV", land)
                g, stage = g + 1, stage + 1
                if stage == n_st:
                    stage, ph = 0, ph ^ 1
            if not ok:
                break
            if slot_readers_release:
                bars[f"LEMPTY{slot}"].arrive()
        if flags["abort"] and "tma_no_drain" not in faults:
            yield drain_copies("tmaK" if is_k else "tmaV")

    def s_issuer():
        kst, kph, sb, su, g = 0, 0, 0, 0, 0
        ok = True
        for it in range(n_items + 1):
            slot = it & 1
            if not (ok := (yield wait(f"LFULL{slot}", (it >> 1) & 1))):
                break
            info = st["info"][slot]
            if info is None:
                break
            _check(info[0] == it, f"S issuer took item {info[0]} for {it}")
            nblk = info[1]
            if slot_readers_release:
                bars[f"LEMPTY{slot}"].arrive()
            if not (ok := (yield wait("QFULL", it & 1))):
                break
            _check(st["Q"] == it, "S reads a stale Q")
            if nblk == 0:
                later("S", lambda it=it: (st.__setitem__("q_free", it), bars["QEMPTY"].arrive()))
            for j in range(nblk):
                if not (ok := (yield wait(f"KFULL{kst}", kph))):
                    break
                _check(st["K"][kst] == g, f"S({g}) reads K stage {kst} holding {st['K'][kst]}")
                if su > 0 and "s_skips_pv_done" not in faults:   # P of block g - 2 sits in this buffer
                    if not (ok := (yield wait(f"PDONE{sb}", (su - 1) & 1))):
                        break
                _check(min(st["pv_done"]) >= g - S_BUFS, f"S({g}) overwrites P({g - S_BUFS}) before PV read it")

                def land(sb=sb, g=g, kst=kst, last=(j == nblk - 1), it=it):
                    st["S"][sb], st["s_done"] = g, g
                    bars[f"SFULL{sb}"].arrive()
                    bars[f"KEMPTY{kst}"].arrive()
                    if last:
                        st["q_free"] = it
                        bars["QEMPTY"].arrive()
                later("S", land)
                g, kst, sb = g + 1, kst + 1, sb + 1
                if kst == K_STAGES:
                    kst, kph = 0, kph ^ 1
                if sb == S_BUFS:
                    sb, su = 0, su + 1
            if not ok:
                break
        if "mma_no_drain" not in faults:
            yield drain_mmas("S")

    def pv_issuer(w):
        vst, vph, sb, su, g = 0, 0, 0, 0, 0
        ok = True
        for it in range(n_items + 1):
            slot = it & 1
            if not (ok := (yield wait(f"LFULL{slot}", (it >> 1) & 1))):
                break
            info = st["info"][slot]
            if info is None:
                break
            _check(info[0] == it, f"PV{w} took item {info[0]} for {it}")
            nblk = info[1]
            if slot_readers_release:
                bars[f"LEMPTY{slot}"].arrive()
            if not (ok := (yield wait("OFREE", (it & 1) ^ 1))):
                break
            _check(st["epilogue_done"] >= it - 1, f"PV{w} overwrites O before the epilogue of item {it - 1}")
            if nblk == 0:
                later(f"PV{w}", lambda: bars["OFULL"].arrive())
            for j in range(nblk):
                if not (ok := (yield wait(f"VFULL{vst}", vph))):
                    break
                _check(st["V"][vst] == g, f"PV{w}({g}) reads V stage {vst} holding {st['V'][vst]}")
                if not (ok := (yield wait(f"PFULL{w}_{sb}", su & 1))):
                    break
                _check(st["S"][sb] == g, f"PV{w}({g}) reads P in S buffer {sb} holding block {st['S'][sb]}")

                def land(w=w, g=g, vst=vst, sb=sb, last=(j == nblk - 1)):
                    st["pv_done"][w] = g
                    bars[f"PDONE{sb}"].arrive()
                    bars[f"VEMPTY{vst}"].arrive()
                    if last:
                        bars["OFULL"].arrive()
                later(f"PV{w}", land)
                g, vst, sb = g + 1, vst + 1, sb + 1
                if vst == V_STAGES:
                    vst, vph = 0, vph ^ 1
                if sb == S_BUFS:
                    sb, su = 0, su + 1
            if not ok:
                break
        if "mma_no_drain" not in faults:
            yield drain_mmas(f"PV{w}")

    def softmax_warp(sg):
        g = 0
        for it in range(n_items + 1):
            slot = it & 1
            if not (yield wait(f"LFULL{slot}", (it >> 1) & 1)):
                return
            info = st["info"][slot]
            if info is None:
                return
            _check(info[0] == it, f"softmax took item {info[0]} for {it}")
            for j in range(info[1]):
                sbuf = g % S_BUFS
                if not (yield wait(f"SFULL{sbuf}", ((g // S_BUFS) + ("softmax_parity" in faults)) & 1)):
                    return
                _check(st["S"][sbuf] == g, f"softmax block {g} reads S buffer holding {st['S'][sbuf]}")
                if hold and g == 0 and not (yield wait("HOLD", 0)):
                    return
                if j > 0 and rng.random() < 0.2:   # the O rescale waits for its previous PV
                    if not (yield wait(f"PDONE{(g - 1) % S_BUFS}", ((g - 1) // S_BUFS) & 1)):
                        return
                    _check(st["pv_done"][sg] >= g - 1, "O rescaled while the previous PV accumulates")
                bars[f"PFULL{sg}_{sbuf}"].arrive()
                g += 1
            if not (yield wait("OFULL", it & 1)):
                return
            _check(info[1] == 0 or min(st["pv_done"]) >= g - 1, "epilogue before the item's last PV")
            bars["LX"].arrive()
            if not (yield wait("LX", it & 1)):
                return
            st["epi"][it] = st["epi"].get(it, 0) + 1
            if st["epi"][it] == 8:
                st["epilogue_done"] = it
            bars["OFREE"].arrive()
            bars[f"LEMPTY{slot}"].arrive()

    roles = {"scheduler": scheduler(), "producer K": producer(True), "producer V": producer(False),
             "S issuer": s_issuer(), "PV0": pv_issuer(0), "PV1": pv_issuer(1)}
    for sg in range(2):
        for wi in range(4):
            roles[f"softmax {sg}.{wi}"] = softmax_warp(sg)
    waiting = {}
    timed_out = []

    def step(name, value):
        try:
            waiting[name] = roles[name].send(value)
        except StopIteration:
            waiting[name] = None

    def resume_value(name):
        """True: the wait returns true; False: it gives up (abort); None: still waiting."""
        kind, arg = waiting[name]
        if kind == "copies":
            return True if not any(iss == arg for iss, _ in pending) else None
        if kind == "drain":
            return True if bars["DRAIN"].passed(arg) else None    # drain waits ignore the abort flag
        if bars[kind].passed(arg):
            return True
        return False if flags["abort"] else None

    for name in roles:
        step(name, None)
    for _ in range(max_steps):
        live = [k for k, v in waiting.items() if v is not None]
        if not live:
            # every thread has reached the end of the kernel: TMEM is freed, the CTA exits
            _check(not pending, "the CTA ends with copies or MMAs in flight: " + ", ".join(i for i, _ in pending))
            return "ok" if not flags["abort"] else "aborted: " + timed_out[0]
        if not flags["abort"] and timeout_p and rng.random() < timeout_p:
            blocked = [k for k in live if resume_value(k) is None]
            if blocked:                     # a wait runs out with work still in flight
                k = rng.choice(blocked)
                timed_out.append(f"{k} waits {waiting[k][0]} parity {waiting[k][1]} (early)")
                flags["abort"] = True
        ready = [("role", k) for k in live if resume_value(k) is not None]
        issuers = list(dict.fromkeys(iss for iss, _ in pending))
        choices = ready + [("done", i) for i in issuers]
        preferred = [c for c in choices if c[1] not in starve]
        choices = preferred or choices
        if not choices:
            stuck = "; ".join(f"{k} waits {waiting[k][0]} parity {waiting[k][1]}" for k in live)
            if flags["abort"]:
                return "deadlock after abort: " + stuck
            # nothing can move: one bounded wait runs out and raises the abort flag
            timed_out.append(stuck)
            flags["abort"] = True
            continue
        kind, who = rng.choice(choices)
        if kind == "role":
            step(who, resume_value(who))
        else:
            idx = next(i for i, (iss, _) in enumerate(pending) if iss == who)
            pending.pop(idx)[1]()
    return "step limit"


def random_items(rng, allow_empty):
    choices = [0, 1, 1, 2, 3, 5, 8] if allow_empty else [1, 1, 2, 3, 5, 8]
    return [rng.choice(choices) for _ in range(rng.randint(1, 7))]
