"""A randomized model of the attention kernel's mbarrier protocol (test
infrastructure; it shares no code with the kernel).

Each role of the kernel (producer, S issuer, P V issuer, the two softmax
groups, the epilogue warpgroup) is a generator that takes the same barrier
waits and arrivals, in the same order, as its counterpart in
csrc/attn_fwd.cuh; the tensor-core and TMA engines are queues that complete
after random delays.  An mbarrier is a phase counter: a parity wait passes
when the completed-phase count has the other parity.  The model checks that

- every parity wait that passes has truly completed the phase it waits for
  (no aliasing: the waiter is never two phases behind);
- no wait is stuck on a phase that is already complete;
- nothing deadlocks;
- no buffer is overwritten before its reader is done (S, P, the
  reference-max exchange, the unit hand-over slots, the O accumulator across
  units), and O is rescaled only once P V of the previous tile has landed.

`two_producers` splits the TMA producer into a K (and Q) warp and a V warp,
each walking the tiles on its own (a variant that was once tried).

`Config.one_s` (BF16 with Dqk 128) models one S buffer taken by the two
groups in turns, with Q copied from its shared-memory slot into tensor
memory at each unit's first tile: the copy is a queue entry in order with
the S MMAs, must find its own unit's Q in the slot, and every S MMA must
find its unit's Q in tensor memory.  Each group waits for the other group's
max of the previous tile before its wait on S.

`run_wide` models the FP8 kernel with 256-key tiles (csrc/attn_fwd_wide.cuh):
one S buffer and one P buffer, both softmax groups on every tile (each on
its own 128-key half), the tile max exchanged through a two-slot buffer under
one barrier both groups arrive on, and the hand-over written by group 0.
It also takes the kernel's two early, non-blocking tests (the next tile's
S, the P buffer), each checked for aliasing when it passes.

`mutation` plants a known mistake, for the tests that show the model catches it.
"""
import random
from dataclasses import dataclass


@dataclass(frozen=True)
class Config:
    stk: int      # K ring stages
    stv: int      # V ring stages
    qbuf: int     # Q tile buffers
    npb: int      # P buffers
    fp8: bool     # FP8 or BF16 (the same protocol)
    hand: int = 8  # unit hand-over slots (and their barriers)
    lead: int = 0  # K tiles the producer keeps ahead of V (0: stk - stv + 1)
    one_s: bool = False  # one S buffer, Q copied into TMEM at each unit's first tile

    @property
    def klead(self):
        return self.lead or self.stk - self.stv + 1


# the kernel's three instantiations
FP8 = Config(stk=4, stv=4, qbuf=2, npb=3, fp8=True)
BF16_D128 = Config(stk=3, stv=2, qbuf=1, npb=2, fp8=False, lead=3, one_s=True)
BF16_D192 = Config(stk=2, stv=2, qbuf=1, npb=2, fp8=False, lead=2)


class ProtocolError(AssertionError):
    pass


class _Bar:
    def __init__(self, name, count):
        self.name, self.count, self.pend, self.c = name, count, 0, 0

    def arrive(self, n=1):
        self.pend += n
        if self.pend > self.count:
            raise ProtocolError(f"{self.name}: more arrivals than expected")
        if self.pend == self.count:
            self.pend = 0
            self.c += 1


def run(units, cfg: Config, seed: int, mutation=None, p_rescale=0.5, two_producers=False):
    """Simulate one CTA that processes `units` (KV-tile counts per unit)."""
    rng = random.Random(seed)
    bars = {}

    def bar(n, cnt):
        bars[n] = _Bar(n, cnt)

    for i in range(2):
        for n, c in (("QF", 1), ("QE", 1), ("SF", 1), ("SC", 128), ("MX", 128)):
            bar(f"{n}{i}", c)
    for i in range(cfg.npb):
        for n, c in (("PF", 128), ("PE", 1)):
            bar(f"{n}{i}", c)
    for i in range(cfg.hand):
        bar(f"LF{i}", 256)
    bar("OF", 128)
    bar("OFIN", 1)
    for i in range(cfg.stk):
        bar(f"KF{i}", 1); bar(f"KE{i}", 1)
    for i in range(cfg.stv):
        bar(f"VF{i}", 1); bar(f"VE{i}", 1)
    tiles = [(u, j, nkv) for u, nkv in enumerate(units) for j in range(nkv)]
    fifos = {"qk": [], "pv": []}
    tma = []
    st = {"P": {}, "O_unit": None, "pv_done": set(), "qk_done": set(), "Sread": {}, "xch": {}, "hand": {},
          "Qsmem": {}, "Qtmem": None}

    def wait(name, parity, need):
        b = bars[name]
        while True:
            passed = (b.c & 1) != parity
            truly = b.c > need
            if passed:
                if not truly:
                    raise ProtocolError(f"aliasing on {name}: parity {parity} passed at phase count {b.c}, "
                                        f"needs more than {need}")
                return
            if truly:
                raise ProtocolError(f"stuck on {name}: phase {need} complete but parity {parity} fails")
            yield "wait"

    def load_k(g):
        u, j, nkv = tiles[g]
        if j == 0:
            slot, n = u % cfg.qbuf, u // cfg.qbuf
            if n > 0:
                yield from wait(f"QE{slot}", (n - 1) & 1, n - 1)
            tma.append([rng.randint(5, 40), f"QF{slot}", ("Q", slot, u)])
        s_, n = g % cfg.stk, g // cfg.stk
        if n > 0:
            yield from wait(f"KE{s_}", (n - 1) & 1, n - 1)
        tma.append([rng.randint(5, 40), f"KF{s_}"])

    def load_v(g):
        s_, n = g % cfg.stv, g // cfg.stv
        if n > 0:
            yield from wait(f"VE{s_}", (n - 1) & 1, n - 1)
        tma.append([rng.randint(5, 40), f"VF{s_}"])

    def producer():
        ks = vs = 0
        for _ in range(cfg.klead):
            if ks < len(tiles):
                yield from load_k(ks); ks += 1
        while vs < len(tiles):
            if ks < len(tiles):
                yield from load_k(ks); ks += 1
            yield from load_v(vs); vs += 1
            yield "step"

    def producer_k():
        for g in range(len(tiles)):
            yield from load_k(g)
            yield "step"

    def producer_v():
        for g in range(len(tiles)):
            yield from load_v(g)
            yield "step"

    def qk_issuer():
        for g, (u, j, nkv) in enumerate(tiles):
            slot = u % cfg.qbuf
            if j == 0:
                yield from wait(f"QF{slot}", (u // cfg.qbuf) & 1, u // cfg.qbuf)
            s_, buf = g % cfg.stk, (0 if cfg.one_s else g & 1)
            yield from wait(f"KF{s_}", (g // cfg.stk) & 1, g // cfg.stk)
            back = 1 if cfg.one_s else 2        # tiles per S buffer
            if g >= back and mutation != "no_sc_wait":
                n = g // back - 1 if not cfg.one_s else g - 1
                yield from wait(f"SC{buf}", n & 1, n)
            if g >= back and st["Sread"].get(buf, -1) < g - back:
                raise ProtocolError(f"S buffer {buf} overwritten by tile {g} before tile {g - back} read it")
            if cfg.one_s:
                if j == 0:
                    # the unit's Q copied from its shared-memory slot into TMEM,
                    # in order with the MMAs; the slot is free once it is done
                    if mutation == "q_slot_freed_before_copy":
                        fifos["qk"].append([0, "commit", [f"QE{slot}"]])
                    fifos["qk"].append([rng.randint(3, 12), "cp", (u, slot)])
                    if mutation != "q_slot_freed_before_copy":
                        fifos["qk"].append([0, "commit", [f"QE{slot}"]])
                fifos["qk"].append([rng.randint(5, 30), "qk", g])
                fifos["qk"].append([0, "commit", [f"SF{buf}", f"KE{s_}"]])
            else:
                fifos["qk"].append([rng.randint(5, 30), "qk", g])
                fifos["qk"].append([0, "commit", [f"SF{buf}", f"KE{s_}"] + ([f"QE{slot}"] if j == nkv - 1 else [])])
            yield "step"

    def pv_issuer():
        for g, (u, j, nkv) in enumerate(tiles):
            s_, buf = g % cfg.stv, g % cfg.npb
            if j == 0 and u > 0:
                yield from wait("OF", (u - 1) & 1, u - 1)
            yield from wait(f"VF{s_}", (g // cfg.stv) & 1, g // cfg.stv)
            yield from wait(f"PF{buf}", (g // cfg.npb) & 1, g // cfg.npb)
            if st["P"].get(buf) != g:
                raise ProtocolError(f"P buffer {buf} holds tile {st['P'].get(buf)} at P V of tile {g}")
            if j == 0:
                if st["O_unit"] not in (None, "free"):
                    raise ProtocolError(f"O still in use by unit {st['O_unit']} at unit {u}")
                st["O_unit"] = u
            fifos["pv"].append([rng.randint(5, 30), "pv", g])
            fifos["pv"].append([0, "commit", [f"VE{s_}", f"PE{buf}"] + (["OFIN"] if j == nkv - 1 else [])])
            yield "step"

    def softmax_group(grp):
        for g, (u, j, nkv) in enumerate(tiles):
            if (g & 1) == grp:
                if cfg.one_s and g >= 1 and mutation != "mx_after_sf":
                    # one S buffer: the other group's max of tile g-1 (published
                    # after it read S of tile g-1) keeps this wait on S at most
                    # one phase behind
                    pb = (g - 1) & 1
                    yield from wait(f"MX{pb}", ((g - 1) >> 1) & 1, (g - 1) >> 1)
                buf = 0 if cfg.one_s else grp
                n = g if cfg.one_s else g >> 1
                yield from wait(f"SF{buf}", n & 1, n)
                if g not in st["qk_done"]:
                    raise ProtocolError(f"S of tile {g} read before its MMA finished")
                yield "load"
                st["Sread"][buf] = g               # the whole row in registers: S released at once
                bars[f"SC{buf}"].arrive(128)
                yield "max"
                if g >= 1:
                    pb = (g - 1) & 1
                    if not cfg.one_s or mutation == "mx_after_sf":
                        yield from wait(f"MX{pb}", ((g - 1) >> 1) & 1, (g - 1) >> 1)
                    if st["xch"].get(pb) != g - 1:
                        raise ProtocolError(f"reference max of tile {g - 1} overwritten before tile {g} read it")
                st["xch"][grp] = g
                bars[f"MX{grp}"].arrive(128)
                pbuf = g % cfg.npb
                back = 2 if mutation == "pe_wait_two_back" else cfg.npb
                if g >= back:
                    yield from wait(f"PE{pbuf}", ((g - back) // cfg.npb) & 1, (g - back) // cfg.npb)
                if g >= cfg.npb and (g - cfg.npb) not in st["pv_done"]:
                    raise ProtocolError(f"P buffer {pbuf} rewritten by tile {g} before P V of tile {g - cfg.npb}")
                for _ in range(rng.randint(0, 4)):
                    yield "codes"
                st["P"][pbuf] = g
                if j > 0 and rng.random() < p_rescale:
                    # the reference max moved: O holds tiles 0 .. g-1 and is rescaled
                    pg = g - 1
                    if mutation != "no_rescale_wait":
                        yield from wait(f"PE{pg % cfg.npb}", (pg // cfg.npb) & 1, pg // cfg.npb)
                    if pg not in st["pv_done"]:
                        raise ProtocolError(f"O rescaled for tile {g} before P V of tile {pg} finished")
                    yield "rescale"
                bars[f"PF{pbuf}"].arrive(128)
            if j == nkv - 1:
                # the unit's last tile: this group's hand-over to the epilogue
                hs = u % cfg.hand
                prev = st["hand"].get((hs, grp))
                if prev is not None and prev != u and prev not in st.setdefault("hand_read", set()):
                    raise ProtocolError(f"hand-over slot {hs} of unit {prev} overwritten by unit {u} before "
                                        f"the epilogue read it")
                st["hand"][(hs, grp)] = u
                bars[f"LF{hs}"].arrive(128)

    def epilogue():
        g_end = 0
        for u, nkv in enumerate(units):
            g_end += nkv
            yield from wait("OFIN", u & 1, u)
            if not all(t in st["pv_done"] for t in range(g_end - nkv, g_end)):
                raise ProtocolError(f"epilogue of unit {u} before its last P V finished")
            hs = u % cfg.hand
            yield from wait(f"LF{hs}", (u // cfg.hand) & 1, u // cfg.hand)
            for grp in (0, 1):
                if st["hand"].get((hs, grp)) != u:
                    raise ProtocolError(f"hand-over of unit {u} (group {grp}) overwritten before the epilogue read it")
            for _ in range(rng.randint(0, 3)):
                yield "epilogue"
            st.setdefault("hand_read", set()).add(u)
            for _ in range(rng.randint(1, 8)):
                yield "epilogue"
            st["O_unit"] = "free"
            bars["OF"].arrive(128)

    roles = {"qk": qk_issuer(), "pv": pv_issuer(), "softmax0": softmax_group(0),
             "softmax1": softmax_group(1), "epilogue": epilogue()}
    if two_producers:
        roles["producer_k"] = producer_k()
        roles["producer_v"] = producer_v()
    else:
        roles["producer"] = producer()
    done, idle = set(), 0
    while len(done) < len(roles):
        progressed = False
        for fk in rng.sample(["qk", "pv"], 2):     # the tensor core completes each issuer's work in order
            f = fifos[fk]
            if not f:
                continue
            e = f[0]
            if e[1] == "commit":
                for n in e[2]:
                    bars[n].arrive()
                f.pop(0)
            else:
                e[0] -= 1
                if e[0] <= 0:
                    if e[1] == "cp":
                        u_, slot_ = e[2]
                        if st["Qsmem"].get(slot_) != u_:
                            raise ProtocolError(f"Q of unit {u_} copied to TMEM from slot {slot_} holding unit "
                                                f"{st['Qsmem'].get(slot_)}")
                        st["Qtmem"] = u_
                    else:
                        if e[1] == "qk" and cfg.one_s and st["Qtmem"] != tiles[e[2]][0]:
                            raise ProtocolError(f"S of tile {e[2]} computed with the Q of unit {st['Qtmem']}")
                        (st["qk_done"] if e[1] == "qk" else st["pv_done"]).add(e[2])
                    f.pop(0)
            progressed = True
        for t in list(tma):
            t[0] -= 1
            if t[0] <= 0:
                if len(t) > 2:
                    _, slot_, u_ = t[2]
                    st["Qsmem"][slot_] = u_
                bars[t[1]].arrive()
                tma.remove(t)
            progressed = True
        names = [n for n in roles if n not in done]
        rng.shuffle(names)
        for n in names:
            try:
                if next(roles[n]) != "wait":
                    progressed = True
            except StopIteration:
                done.add(n)
                progressed = True
        idle = 0 if progressed else idle + 1
        if idle >= 1000:
            raise ProtocolError("deadlock: " + ", ".join(f"{k} {b.c}/{b.pend}" for k, b in bars.items() if b.pend))


@dataclass(frozen=True)
class WideConfig:
    stk: int = 3   # K ring stages (256-key tiles)
    stv: int = 2   # V ring stages
    qbuf: int = 2  # Q tile buffers
    hand: int = 8  # unit hand-over slots

    @property
    def klead(self):
        return self.stk - self.stv + 1


WIDE = WideConfig()


def run_wide(units, cfg: WideConfig, seed: int, mutation=None, p_rescale=0.5):
    """Simulate one CTA of the 256-key-tile kernel over `units` (tile counts)."""
    rng = random.Random(seed)
    bars = {}

    def bar(n, cnt):
        bars[n] = _Bar(n, cnt)

    for i in range(cfg.qbuf):
        bar(f"QF{i}", 1); bar(f"QE{i}", 1)
    for n, c in (("SF", 1), ("SC", 256), ("MXA", 256), ("PF", 256), ("PE", 1), ("OF", 128), ("OFIN", 1)):
        bar(n, c)
    for i in range(cfg.hand):
        bar(f"LF{i}", 128)
    for i in range(cfg.stk):
        bar(f"KF{i}", 1); bar(f"KE{i}", 1)
    for i in range(cfg.stv):
        bar(f"VF{i}", 1); bar(f"VE{i}", 1)
    tiles = [(u, j, nkv) for u, nkv in enumerate(units) for j in range(nkv)]
    # the rescale decision of a tile: both groups compute the same one
    rescale = [j > 0 and rng.random() < p_rescale for (u, j, nkv) in tiles]
    fifos = {"qk": [], "pv": []}
    tma = []
    st = {"P": {}, "O_unit": None, "pv_done": set(), "qk_done": set(), "Sread": {0: -1, 1: -1},
          "xch": {}, "xch_read": {}, "hand": {}, "hand_read": set()}

    def wait(name, parity, need):
        b = bars[name]
        while True:
            passed = (b.c & 1) != parity
            truly = b.c > need
            if passed:
                if not truly:
                    raise ProtocolError(f"aliasing on {name}: parity {parity} passed at phase count {b.c}, "
                                        f"needs more than {need}")
                return
            if truly:
                raise ProtocolError(f"stuck on {name}: phase {need} complete but parity {parity} fails")
            yield "wait"

    def test(name, parity, need):
        """Non-blocking test of a phase (test_wait): True when it passes."""
        b = bars[name]
        if (b.c & 1) != parity:
            if b.c <= need:
                raise ProtocolError(f"aliasing on {name}: early test of parity {parity} passed at phase count "
                                    f"{b.c}, needs more than {need}")
            return True
        return False

    def producer():
        def load_k(g):
            u, j, nkv = tiles[g]
            if j == 0:
                slot, n = u % cfg.qbuf, u // cfg.qbuf
                if n > 0:
                    yield from wait(f"QE{slot}", (n - 1) & 1, n - 1)
                tma.append([rng.randint(5, 40), f"QF{slot}"])
            s_, n = g % cfg.stk, g // cfg.stk
            if n > 0:
                yield from wait(f"KE{s_}", (n - 1) & 1, n - 1)
            tma.append([rng.randint(5, 40), f"KF{s_}"])

        def load_v(g):
            s_, n = g % cfg.stv, g // cfg.stv
            if n > 0:
                yield from wait(f"VE{s_}", (n - 1) & 1, n - 1)
            tma.append([rng.randint(5, 40), f"VF{s_}"])

        ks = vs = 0
        for _ in range(cfg.klead):
            if ks < len(tiles):
                yield from load_k(ks); ks += 1
        while vs < len(tiles):
            if ks < len(tiles):
                yield from load_k(ks); ks += 1
            yield from load_v(vs); vs += 1
            yield "step"

    def qk_issuer():
        for g, (u, j, nkv) in enumerate(tiles):
            slot = u % cfg.qbuf
            if j == 0:
                yield from wait(f"QF{slot}", (u // cfg.qbuf) & 1, u // cfg.qbuf)
            s_ = g % cfg.stk
            yield from wait(f"KF{s_}", (g // cfg.stk) & 1, g // cfg.stk)
            if g >= 1 and mutation != "no_sc_wait":
                yield from wait("SC", (g - 1) & 1, g - 1)
            if g >= 1 and min(st["Sread"].values()) < g - 1:
                raise ProtocolError(f"S overwritten by tile {g} before both groups read tile {g - 1}")
            fifos["qk"].append([rng.randint(5, 30), "qk", g])
            fifos["qk"].append([0, "commit", ["SF", f"KE{s_}"] + ([f"QE{slot}"] if j == nkv - 1 else [])])
            yield "step"

    def pv_issuer():
        for g, (u, j, nkv) in enumerate(tiles):
            s_ = g % cfg.stv
            if j == 0 and u > 0:
                yield from wait("OF", (u - 1) & 1, u - 1)
            yield from wait(f"VF{s_}", (g // cfg.stv) & 1, g // cfg.stv)
            yield from wait("PF", g & 1, g)
            if st["P"].get(0) != g or st["P"].get(1) != g:
                raise ProtocolError(f"P holds tiles {st['P']} at P V of tile {g}")
            if j == 0:
                if st["O_unit"] not in (None, "free"):
                    raise ProtocolError(f"O still in use by unit {st['O_unit']} at unit {u}")
                st["O_unit"] = u
            fifos["pv"].append([rng.randint(5, 30), "pv", g])
            fifos["pv"].append([0, "commit", [f"VE{s_}", "PE"] + (["OFIN"] if j == nkv - 1 else [])])
            yield "step"

    def softmax_group(x):
        sf_t = False        # S of the next tile seen complete by the early test
        for g, (u, j, nkv) in enumerate(tiles):
            if not sf_t:
                yield from wait("SF", g & 1, g)
            if g not in st["qk_done"]:
                raise ProtocolError(f"S of tile {g} read before its MMA finished")
            yield "load"
            st["Sread"][x] = g
            bars["SC"].arrive(128)
            yield "max"
            slot = g & 1
            prev = st["xch"].get((slot, x))
            if prev is not None and st["xch_read"].get((slot, x)) != prev:
                raise ProtocolError(f"tile max of tile {prev} (group {x}) overwritten before the other group read it")
            st["xch"][(slot, x)] = g
            bars["MXA"].arrive(128)
            if mutation != "no_mx_wait":
                yield from wait("MXA", g & 1, g)
            if st["xch"].get((slot, 1 - x)) != g:
                raise ProtocolError(f"group {x} read the other group's tile max of tile "
                                    f"{st['xch'].get((slot, 1 - x))} at tile {g}")
            st["xch_read"][(slot, 1 - x)] = g
            # the P buffer, tested before the codes and waited for after them
            pe_t = g < 1 or test("PE", (g - 1) & 1, g - 1)
            for _ in range(rng.randint(0, 4)):
                yield "codes"
            if g >= 1 and not pe_t and mutation != "no_pe_wait":
                yield from wait("PE", (g - 1) & 1, g - 1)
            if g >= 1 and (g - 1) not in st["pv_done"]:
                raise ProtocolError(f"P or O touched for tile {g} before P V of tile {g - 1} finished")
            if rescale[g]:
                yield "rescale"
            # S of the next tile, tested before this tile's P store
            sf_t = test("SF", (g + (2 if mutation == "early_sf_two_ahead" else 1)) & 1, g + 1)
            st["P"][x] = g
            bars["PF"].arrive(128)
            if j == nkv - 1 and x == 0:
                hs = u % cfg.hand
                prev = st["hand"].get(hs)
                if prev is not None and prev not in st["hand_read"]:
                    raise ProtocolError(f"hand-over slot {hs} of unit {prev} overwritten by unit {u} before "
                                        f"the epilogue read it")
                st["hand"][hs] = u
                bars[f"LF{hs}"].arrive(128)

    def epilogue():
        g_end = 0
        for u, nkv in enumerate(units):
            g_end += nkv
            yield from wait("OFIN", u & 1, u)
            if not all(t in st["pv_done"] for t in range(g_end - nkv, g_end)):
                raise ProtocolError(f"epilogue of unit {u} before its last P V finished")
            hs = u % cfg.hand
            yield from wait(f"LF{hs}", (u // cfg.hand) & 1, u // cfg.hand)
            if st["hand"].get(hs) != u:
                raise ProtocolError(f"hand-over of unit {u} overwritten before the epilogue read it")
            for _ in range(rng.randint(0, 3)):
                yield "epilogue"
            st["hand_read"].add(u)
            for _ in range(rng.randint(1, 8)):
                yield "epilogue"
            st["O_unit"] = "free"
            bars["OF"].arrive(128)

    roles = {"producer": producer(), "qk": qk_issuer(), "pv": pv_issuer(), "softmax0": softmax_group(0),
             "softmax1": softmax_group(1), "epilogue": epilogue()}
    done, idle = set(), 0
    while len(done) < len(roles):
        progressed = False
        for fk in rng.sample(["qk", "pv"], 2):
            f = fifos[fk]
            if not f:
                continue
            e = f[0]
            if e[1] == "commit":
                for n in e[2]:
                    bars[n].arrive()
                f.pop(0)
            else:
                e[0] -= 1
                if e[0] <= 0:
                    (st["qk_done"] if e[1] == "qk" else st["pv_done"]).add(e[2])
                    f.pop(0)
            progressed = True
        for t in list(tma):
            t[0] -= 1
            if t[0] <= 0:
                bars[t[1]].arrive()
                tma.remove(t)
            progressed = True
        names = [n for n in roles if n not in done]
        rng.shuffle(names)
        for n in names:
            try:
                if next(roles[n]) != "wait":
                    progressed = True
            except StopIteration:
                done.add(n)
                progressed = True
        idle = 0 if progressed else idle + 1
        if idle >= 1000:
            raise ProtocolError("deadlock: " + ", ".join(f"{k} {b.c}/{b.pend}" for k, b in bars.items() if b.pend))


def random_units(rng):
    """KV-tile counts of the units one CTA takes: random lengths, or (as the
    heaviest-first queue hands them out) descending, ending in runs of
    one-tile units."""
    units = [rng.randint(1, 7) if rng.random() < 0.6 else 1 for _ in range(rng.randint(1, 12))]
    if rng.random() < 0.5:
        units.sort(reverse=True)
    return units
