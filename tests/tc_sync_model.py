"""A checkable model of how the tensor-core scan kernels synchronise their roles.

Both kernels in ``state_space_model_07_b200/csrc/ssd_tc.cu`` split one CTA into
warp roles that hand buffers (shared-memory stages, TMEM regions) to one another
through mbarriers, while TMA copies and tcgen05 MMAs run asynchronously to the
threads that issued them.  Whether that hand-off protocol is free of data races,
deadlocks and parity aliasing is an argument about orderings, which a GPU run
can confirm only for the schedules the hardware happened to take.  This module
restates each role's sequence of barrier operations and buffer accesses (per
tile, in program order, as the kernel source has them) and runs the roles
under many random schedules, checking every one:

* mbarriers follow the PTX phase rules: a phase completes when its pending
  arrival count and its transaction count both reach zero; ``try_wait.parity``
  passes when the phase of the given parity has completed, i.e. when the
  number of completed phases and the parity differ in their low bit.  Each
  wait in the model names the phase index it means; a wait that passes on any
  other phase (a barrier two phases ahead of, or behind, its waiter) is
  reported as aliasing.
* async engines: each TMA load completes on its own, in any order, and then
  counts its bytes down on its barrier; tcgen05 operations of one issuing
  thread run in issue order, and ``tcgen05.commit`` arrives on its barrier
  once all earlier operations of that thread are done; a TMA store's
  shared-memory reads finish at the issuer's ``wait_group.read``.
* happens-before is tracked with vector clocks (arrivals release, passed
  waits acquire; an async operation inherits its issuer's clock at issue), and
  every buffer access is checked against the conflicting accesses before it
  (two accesses conflict when one is a write and neither happens before the
  other).
* at CTA exit (all roles done) no TMA copy or tensor-core operation may still
  be in flight (the kernel frees TMEM there).
* the timeout path: a run may time out one waiting role at a random step.
  Every copy and MMA issued before then completes first, since a timeout
  takes hundreds of milliseconds.  The CTA then gives up: later waits fail at
  once, as the kernel's wait_bar does when the abort flag is set, and each
  role leaves its loop the way the kernel does.  From there on only deadlock
  and exit with work in flight are checked.

A role whose warps always meet at a named barrier before each mbarrier wait
(the kernel's leader-polls-then-``bar.sync`` waits) moves as one agent; its
per-warp arrivals are one arrival of the role's warp count.
"""
from __future__ import annotations

import random
from dataclasses import dataclass, field


class ProtocolError(AssertionError):
    pass


def _join(a: dict, b: dict) -> dict:
    out = dict(a)
    for k, v in b.items():
        if out.get(k, 0) < v:
            out[k] = v
    return out


class Barrier:
    def __init__(self, name: str, count: int):
        self.name, self.count = name, count
        self.pending, self.tx, self.completed = count, 0, 0
        self.acc: dict = {}
        self.phase_vc: list = []

    def _release(self, vc):
        self.acc = _join(self.acc, vc)

    def arrive(self, vc, weight=1, tx=0):
        self._release(vc)
        self.tx += tx
        self.pending -= weight
        if self.pending < 0:
            raise ProtocolError(f"{self.name}: more arrivals than its count in phase {self.completed}")
        self._maybe_complete()

    def complete_tx(self, vc, nbytes=1):
        self._release(vc)
        self.tx -= nbytes
        self._maybe_complete()

    def _maybe_complete(self):
        if self.pending == 0 and self.tx == 0:
            self.phase_vc.append(self.acc)
            self.completed += 1
            self.pending, self.acc = self.count, {}

    def try_wait(self, phase: int, strict: bool = True):
        """(passed, vc) for a wait meant for phase index `phase` (parity phase & 1).  A strict
        wait (the protocol's own) must pass on exactly that phase; a drain on the timeout path
        only asks whether the parity has flipped."""
        passed = (self.completed & 1) != (phase & 1)
        if not strict:
            return passed, (self.phase_vc[-1] if passed else None)
        if passed:
            if self.completed != phase + 1:
                raise ProtocolError(f"{self.name}: wait for phase {phase} passed with {self.completed} "
                                    f"phases complete (parity aliasing)")
            return True, self.phase_vc[phase]
        if self.completed >= phase + 2:
            raise ProtocolError(f"{self.name}: barrier ran two phases past a waiter for phase {phase}")
        return False, None


@dataclass
class _Buf:
    write: tuple | None = None                     # (component, clock, who)
    reads: list = field(default_factory=list)


class Machine:
    """One CTA: barriers, buffers, role agents and async engines."""

    def __init__(self):
        self.bars: dict[str, Barrier] = {}
        self.bufs: dict[str, _Buf] = {}
        self.agents: dict[str, dict] = {}
        self.tc_queues: dict[str, list] = {}       # issuer -> in-order tcgen05 ops
        self.tc_last: dict[str, dict] = {}
        self.bulk_queues: dict[str, list] = {}     # issuer -> in-order TMA store reads
        self.bulk_last: dict[str, dict] = {}
        self.tma_loads: list = []                  # independent in-flight loads
        self.nop = 0
        self.abort = False                         # a bounded wait has timed out
        self.races = True                          # race checks (off once the CTA is giving up)

    # ---- declarations
    def barrier(self, name, count):
        self.bars[name] = Barrier(name, count)

    def role(self, name, gen):
        self.agents[name] = {"gen": gen, "op": None, "done": False, "vc": {name: 1}, "send": None}
        self.tc_queues[name], self.bulk_queues[name] = [], []
        self.tc_last[name], self.bulk_last[name] = {}, {}

    # ---- accesses and happens-before
    @staticmethod
    def _hb(epoch, vc):
        return vc.get(epoch[0], 0) >= epoch[1]

    def _access(self, buf, kind, epoch, vc, who):
        if not self.races:
            return
        b = self.bufs.setdefault(buf, _Buf())
        if b.write is not None and not self._hb(b.write, vc):
            raise ProtocolError(f"race on {buf}: {who} {kind}s it unordered with a write by {b.write[2]}")
        if kind == "write":
            for r in b.reads:
                if not self._hb(r, vc):
                    raise ProtocolError(f"race on {buf}: {who} writes it unordered with a read by {r[2]}")
            b.write, b.reads = epoch, []
        else:
            b.reads.append(epoch)

    def _async_vc(self, base):
        self.nop += 1
        cid = ("op", self.nop)
        vc = dict(base)
        vc[cid] = 1
        return vc, (cid, 1)

    # ---- one step of an agent
    def _fetch(self, a):
        if a["op"] is None and not a["done"]:
            try:
                a["op"] = a["gen"].send(a["send"])
            except StopIteration:
                a["done"] = True
            a["send"] = None

    def _progress_possible(self, bar):
        """Whether async work in flight can still complete a phase of `bar`."""
        return (any(ld[0] == bar for ld in self.tma_loads)
                or any(op[0] == "commit" and op[1] == bar for q in self.tc_queues.values() for op, _ in q))

    def _runnable(self, name):
        a = self.agents[name]
        self._fetch(a)
        if a["done"]:
            return False
        op = a["op"]
        if op[0] == "wait":
            # the kernel's wait_bar gives up at once when the CTA is aborting
            return self.abort or self.bars[op[1]].try_wait(op[2])[0]
        if op[0] == "bwait":
            # a bounded wait that ignores the abort flag: passes on the parity, or times out
            # once nothing in flight can complete the phase
            return self.bars[op[1]].try_wait(op[2], strict=False)[0] or not self._progress_possible(op[1])
        if op[0] == "store_wait":
            return not self.bulk_queues[name]
        return True

    def _drain_async(self):
        """A timeout takes hundreds of milliseconds, which every copy and MMA issued before it
        outlasts: they all complete first."""
        while self.tma_loads:
            self._step_tma(0)
        for n in self.tc_queues:
            while self.tc_queues[n]:
                self._step_tc(n)
        for n in self.bulk_queues:
            while self.bulk_queues[n]:
                self._step_bulk(n)

    def _fault(self, rng):
        """Times out one role that is waiting; the CTA starts giving up."""
        waiting = [n for n, a in self.agents.items() if not a["done"] and a["op"] is not None
                   and a["op"][0] == "wait"]
        if not waiting:
            return False
        self._drain_async()
        name = rng.choice(waiting)
        self.abort, self.races = True, False
        a = self.agents[name]
        a["op"], a["send"] = None, False
        return True

    def _tick(self, name):
        a = self.agents[name]
        a["vc"] = dict(a["vc"])
        a["vc"][name] += 1

    def _step_agent(self, name):
        a = self.agents[name]
        op, vc = a["op"], a["vc"]
        kind = op[0]
        if kind == "wait":
            ok, pvc = self.bars[op[1]].try_wait(op[2], strict=not self.abort)
            if self.abort:
                ok = False           # wait_bar checks the abort flag before it polls
            if ok:
                a["vc"] = _join(vc, pvc)
            a["send"] = ok
        elif kind == "bwait":
            ok, pvc = self.bars[op[1]].try_wait(op[2], strict=False)
            if ok:
                a["vc"] = _join(vc, pvc)
            a["send"] = ok
        elif kind == "store_wait":
            a["vc"] = _join(vc, self.bulk_last[name])
        elif kind == "arrive":
            self.bars[op[1]].arrive(vc, weight=op[2] if len(op) > 2 else 1)
            self._tick(name)
        elif kind == "arrive_tx":
            self.bars[op[1]].arrive(vc, weight=1, tx=op[2])
            self._tick(name)
        elif kind in ("read", "write"):
            for buf in op[1:]:
                self._access(buf, kind, (name, vc[name], name), vc, name)
        elif kind == "tma_load":
            self.tma_loads.append((op[1], op[2], dict(vc)))
            self._tick(name)
        elif kind in ("mma", "commit"):
            self.tc_queues[name].append((op, dict(vc)))
            self._tick(name)
        elif kind == "store":
            self.bulk_queues[name].append((op, dict(vc)))
            self._tick(name)
        else:
            raise ValueError(kind)
        a["op"] = None

    # ---- async engines
    def _step_tma(self, i):
        bar, buf, ivc = self.tma_loads.pop(i)
        vc, ep = self._async_vc(ivc)
        self._access(buf, "write", (ep[0], ep[1], f"TMA load of {buf}"), vc, f"TMA load of {buf}")
        self.bars[bar].complete_tx(vc)

    def _step_tc(self, issuer):
        op, ivc = self.tc_queues[issuer].pop(0)
        vc, ep = self._async_vc(_join(ivc, self.tc_last[issuer]))
        who = f"tcgen05 op of {issuer}"
        if op[0] == "mma":
            reads, writes = op[1], op[2]
            for buf in reads:
                self._access(buf, "read", (ep[0], ep[1], who), vc, who)
            for buf in writes:
                self._access(buf, "write", (ep[0], ep[1], who), vc, who)
        else:
            self.bars[op[1]].arrive(vc)
        self.tc_last[issuer] = vc

    def _step_bulk(self, issuer):
        op, ivc = self.bulk_queues[issuer].pop(0)
        vc, ep = self._async_vc(_join(ivc, self.bulk_last[issuer]))
        who = f"TMA store of {issuer}"
        for buf in op[1]:
            self._access(buf, "read", (ep[0], ep[1], who), vc, who)
        self.bulk_last[issuer] = vc

    # ---- schedule
    def run(self, rng: random.Random, max_steps=1_000_000, fault_at=None):
        """One random schedule.  `fault_at`: the step at which a waiting role times out (the
        first step from there on at which some role waits), None for none."""
        names = list(self.agents)
        weight = {n: 10 ** rng.uniform(-2.5, 0) for n in names}
        w_tma, w_tc, w_bulk = (10 ** rng.uniform(-2.5, 0) for _ in range(3))
        for step in range(max_steps):
            if fault_at is not None and step >= fault_at and not self.abort:
                for n in names:
                    self._fetch(self.agents[n])
                self._fault(rng)
            choices, weights = [], []
            for n in names:
                if self._runnable(n):
                    choices.append(("agent", n))
                    weights.append(weight[n])
            if all(a["done"] for a in self.agents.values()):
                break                               # every role has left: the CTA frees TMEM and exits
            for i in range(len(self.tma_loads)):
                choices.append(("tma", i))
                weights.append(w_tma)
            for n, q in self.tc_queues.items():
                if q:
                    choices.append(("tc", n))
                    weights.append(w_tc)
            for n, q in self.bulk_queues.items():
                if q:
                    choices.append(("bulk", n))
                    weights.append(w_bulk)
            if not choices:
                break
            kind, arg = rng.choices(choices, weights)[0]
            if kind == "agent":
                self._step_agent(arg)
            elif kind == "tma":
                self._step_tma(arg)
            elif kind == "tc":
                self._step_tc(arg)
            else:
                self._step_bulk(arg)
        else:
            raise RuntimeError("schedule did not finish")
        stuck = {n: a["op"] for n, a in self.agents.items() if not a["done"]}
        if stuck:
            raise ProtocolError(f"deadlock: {stuck}")
        if self.tma_loads or any(self.tc_queues.values()) or any(self.bulk_queues.values()):
            raise ProtocolError("CTA exits with TMA copies or tensor-core operations in flight")


# ---------------------------------------------------------------------------
# Role scripts.  Each yields the operations of one role in program order; a
# wait evaluates to True when it passed and False when it gave up (the
# kernel's bounded waits), after which the role leaves its loop as the kernel
# does.  `drop` removes named protocol steps, to show that the checker
# catches each of them.


def _prefixed(gen, pre: str, peer: str):
    """Runs a role script inside one CTA of a cluster: every barrier and buffer name gets the
    CTA's prefix, names written "peer:..." get the other CTA's (distributed shared memory)."""
    nm = lambda x: peer + x[5:] if x.startswith("peer:") else pre + x

    def conv(op):
        k = op[0]
        if k in ("wait", "bwait", "arrive", "arrive_tx", "commit"):
            return (k, nm(op[1])) + tuple(op[2:])
        if k in ("read", "write"):
            return (k,) + tuple(nm(b) for b in op[1:])
        if k == "tma_load":
            return (k, nm(op[1]), nm(op[2]))
        if k == "mma":
            return (k, tuple(nm(b) for b in op[1]), tuple(nm(b) for b in op[2]))
        if k == "store":
            return (k, tuple(nm(b) for b in op[1]))
        return op

    try:
        op = gen.send(None)
        while True:
            val = yield conv(op)
            op = gen.send(val)
    except StopIteration:
        return


# The decoupled-state kernel (k_tc_scan3, d_state 128).  `nt` tiles of 128
# tokens; `partial` = the last tile is shorter (its y leaves by row stores,
# not through the staging tile).

def build_scan3(nt: int, partial: bool = False, drop: frozenset = frozenset(), zero_b: str = "",
                conv: str = "E", m: Machine | None = None, rank: int | None = None,
                y_issuer: bool = False) -> Machine:
    """`zero_b` models ways of zeroing the B rows past the sequence end in a partial last tile
    (not done by the kernel today): "p" has the P warps do it right after C B^T has read B
    (cb_full), with W17 waiting for c_scaled before B^T (w o x) on that tile; "e" has the E
    warps do it before x_ready, unordered with W18's C B^T read.

    `conv` names the role that turns x into the fp16 operands x and w o x: "E" (the kernel
    today: the E warps, between the state update of tile t - 1 and x_ready of tile t) or "Y"
    (a candidate: the four epilogue warps convert x of tile t + 1 as soon as B^T (w o x) of
    tile t has completed, and the E warps do only the state update, which then leaves the loop
    between consecutive B^T (w o x) MMAs), or "Y2" (the same, in two phases: x of tile t + 1 is
    converted in place as soon as it has landed, kept in registers, and only w o x is written
    after B^T (w o x) of tile t), or "E2" (the kernel's form: the E warps convert x of tile
    t + 1 in place while B^T (w o x) of tile t runs, and once it has completed they load s,
    release the s buffer, write w o x of tile t + 1 from the converted x and then the state
    entering tile t + 1).

    `y_issuer` moves the output chain (C' h_prev, then S x into one accumulator) from W17 to a
    warp of its own (W24), as the kernel has it: W17 then issues only B^T (w o x); W24 also waits
    for x_ready, since S x reads the converted x.

    `rank` (0 or 1, with a shared `m`) builds one CTA of the d_state 256 pair candidate (see
    build_scan3_pair): C gets one shared-memory stage on its own barrier, and the epilogues
    exchange Y through distributed shared memory."""
    pre, peer = ("", "") if rank is None else (("a.", "b.") if rank == 0 else ("b.", "a."))
    m = m or Machine()
    reg = lambda name, count: m.barrier(pre + name, count)
    for i in range(4):
        reg(f"scan_done{i}", 1)
        reg(f"scan_free{i}", 16 if conv in ("E", "E2") else 20)
    for i in range(2):
        for name, count in (("full", 1), ("cb_full", 1), ("cb_free", 8), ("c_scaled", 8), ("s_ready", 8),
                            ("x_ready", 8), ("hs_ready", 8), ("e_done", 4), ("stg_free", 1), ("s_done", 1),
                            ("y_full", 1), ("fin", 1), ("st_free", 8), ("rcv_full", 1), ("rcv_free", 1)):
            reg(f"{name}{i}", count if not (name == "x_ready" and conv in ("Y", "Y2")) else 4)
    reg("cfull", 1)
    reg("fin2", 1)
    pair = rank is not None
    full_tile = lambda u: not (partial and u == nt - 1)

    def w19():      # decay scan into the four-slot ring
        for u in range(nt):
            sl = u & 3
            if u >= 4 and "w19_scan_free" not in drop:
                if not (yield ("wait", f"scan_free{sl}", (u - 4) >> 2)):
                    break
            yield ("write", f"ring{sl}")
            yield ("arrive", f"scan_done{sl}")

    def w16():      # TMA loads of x, B, C, two stages
        issued = 0
        for u in range(nt):
            st = u & 1
            if u >= 2 and "w16_y_full" not in drop:
                if not (yield ("wait", f"y_full{st}", (u - 2) >> 1)):
                    break
            if u >= 2 and y_issuer and "w16_s_done" not in drop:
                # B^T (w o x) of tile u - 2 is W17's, not covered by W24's y_full commit
                if not (yield ("wait", f"s_done{st}", (u - 2) >> 1)):
                    break
            yield ("arrive_tx", f"full{st}", 2 if pair else 3)
            for buf in (("x", "b") if pair else ("x", "b", "c")):
                yield ("tma_load", f"full{st}", f"{buf}{st}")
            issued += 1
            if pair:
                # one C stage: free once the copy of C(u - 1) to TMEM has completed
                if u >= 1 and "pair_c_stage" not in drop:
                    if not (yield ("wait", f"cb_full{st ^ 1}", (u - 1) >> 1)):
                        break
                yield ("arrive_tx", "cfull", 1)
                yield ("tma_load", "cfull", "c0")
        if m.abort and "w16_drain" not in drop:
            # let the copies in flight land before the CTA exits
            for u in range(issued):
                yield ("bwait", f"full{u & 1}", u >> 1)
                if pair:
                    yield ("bwait", "cfull", u)

    def w18():      # C -> TMEM copy and C B^T
        if nt == 0:
            return
        for t in range(nt):
            st = t & 1
            if not (yield ("wait", f"full{st}", t >> 1)):
                break
            if t >= 2 and "w18_y_full" not in drop:
                if not (yield ("wait", f"y_full{st}", (t - 2) >> 1)):
                    break
            if pair and not (yield ("wait", "cfull", t)):
                break
            yield ("mma", ("c0" if pair else f"c{st}",), (f"tC{st}",))     # tcgen05.cp
            if t >= 1 and "w18_cb_free" not in drop:
                if not (yield ("wait", f"cb_free{st ^ 1}", (t - 1) >> 1)):
                    break
            yield ("mma", (f"tC{st}", f"b{st}"), ("tCB",))
            yield ("commit", f"cb_full{st}")
        if "w18_fin" not in drop:
            yield ("commit", "fin0")
            yield ("bwait", "fin0", 0)

    def w17():      # s, C' h_prev, S x
        if nt == 0:
            return
        for t in range(nt):
            st, ph = t & 1, t >> 1
            if not (yield ("wait", f"x_ready{st}", ph)) or not (yield ("wait", f"full{st}", ph)):
                break
            if conv != "E" and t >= 1 and "w17_st_free" not in drop:
                # the single s buffer: E has loaded s of tile t - 1
                if not (yield ("wait", f"st_free{st ^ 1}", (t - 1) >> 1)):
                    break
            if zero_b == "p" and not full_tile(t):
                if not (yield ("wait", f"c_scaled{st}", ph)):
                    break
            yield ("mma", (f"b{st}", "wx"), ("tSt",))
            yield ("commit", f"s_done{st}")
            if y_issuer:
                continue
            if not (yield ("wait", f"hs_ready{st}", ph)) or not (yield ("wait", f"c_scaled{st}", ph)):
                break
            if t >= 2 and "w17_e_done" not in drop:
                if not (yield ("wait", f"e_done{st}", (t - 2) >> 1)):
                    break
            yield ("mma", (f"tC{st}", f"hs{st}"), (f"tY{st}",))
            if "w17_s_ready" not in drop:
                if not (yield ("wait", f"s_ready{st}", ph)):
                    break
            yield ("mma", ("tS", f"x{st}", f"tY{st}"), (f"tY{st}",))
            yield ("commit", f"y_full{st}")
        if "w17_fin" not in drop:
            yield ("commit", "fin1")
            yield ("bwait", "fin1", 0)

    def w24():      # the output chain on its own warp: C' h_prev, then S x
        if nt == 0:
            return
        for t in range(nt):
            st, ph = t & 1, t >> 1
            if not (yield ("wait", f"hs_ready{st}", ph)) or not (yield ("wait", f"c_scaled{st}", ph)):
                break
            if t >= 2 and "w17_e_done" not in drop:
                if not (yield ("wait", f"e_done{st}", (t - 2) >> 1)):
                    break
            yield ("mma", (f"tC{st}", f"hs{st}"), (f"tY{st}",))
            if "w17_s_ready" not in drop:
                if not (yield ("wait", f"s_ready{st}", ph)):
                    break
            if "w24_x_ready" not in drop:
                if not (yield ("wait", f"x_ready{st}", ph)):
                    break
            yield ("mma", ("tS", f"x{st}", f"tY{st}"), (f"tY{st}",))
            yield ("commit", f"y_full{st}")
        if "w24_fin" not in drop:
            yield ("commit", "fin2")
            yield ("bwait", "fin2", 0)

    def p_role():   # C' scaling and the decay mask S
        yield ("write", "tS")                       # blocks right of the diagonal, zeroed once
        for t in range(nt):
            st, sl = t & 1, t & 3
            if not (yield ("wait", f"scan_done{sl}", t >> 2)) or not (yield ("wait", f"cb_full{st}", t >> 1)):
                break
            yield ("read", f"ring{sl}", f"tC{st}")
            yield ("write", f"tC{st}")
            if zero_b == "p" and not full_tile(t):
                yield ("write", f"b{st}")
            yield ("arrive", f"c_scaled{st}", 8)
            yield ("read", "tCB", f"ring{sl}")
            yield ("arrive", f"cb_free{st}", 8)
            yield ("arrive", f"scan_free{sl}", 8)
            if t > 0 and "p_y_full" not in drop:
                if not (yield ("wait", f"y_full{st ^ 1}", (t - 1) >> 1)):
                    break
            yield ("write", "tS")
            yield ("arrive", f"s_ready{st}", 8)

    def convert(k, weight):   # x of tile k -> fp16 x and w o x
        if not (yield ("wait", f"scan_done{k & 3}", k >> 2)) or not (yield ("wait", f"full{k & 1}", k >> 1)):
            return False
        yield ("read", f"ring{k & 3}")
        yield ("arrive", f"scan_free{k & 3}", weight)
        yield ("read", f"x{k & 1}")
        yield ("write", f"x{k & 1}", "wx")
        if zero_b == "e" and not full_tile(k):
            yield ("write", f"b{k & 1}")
        yield ("arrive", f"x_ready{k & 1}", weight)
        return True

    def convert_in_place(k):   # phase 1 of "Y2": x of tile k -> fp16 in place (kept in registers)
        if not (yield ("wait", f"scan_done{k & 3}", k >> 2)) or not (yield ("wait", f"full{k & 1}", k >> 1)):
            return False
        yield ("read", f"ring{k & 3}")
        yield ("arrive", f"scan_free{k & 3}", 4)
        yield ("read", f"x{k & 1}")
        yield ("write", f"x{k & 1}")
        return True

    def write_wx(k):           # phase 2 of "Y2": w o x from the registers
        yield ("write", "wx")
        yield ("arrive", f"x_ready{k & 1}", 4)

    def y_role():   # epilogue and TMA store of y
        stored = False
        if conv == "Y" and nt > 0 and not (yield from convert(0, 4)):
            return
        if conv == "Y2" and nt > 0:
            if not (yield from convert_in_place(0)):
                return
            yield from write_wx(0)
        for u in range(nt):
            st = u & 1
            if conv == "Y" and u + 1 < nt:
                # w o x is free once B^T (w o x) of tile u has completed
                if not (yield ("wait", f"s_done{st}", u >> 1)) or not (yield from convert(u + 1, 4)):
                    break
            if conv == "Y2" and u + 1 < nt:
                if not (yield from convert_in_place(u + 1)):
                    break
                if not (yield ("wait", f"s_done{st}", u >> 1)):
                    break
                yield from write_wx(u + 1)
            if not (yield ("wait", f"y_full{st}", u >> 1)):
                break
            yield ("read", f"tY{st}")
            if rank == 1:
                # the second CTA hands its fp32 Y partial to the first one's shared memory
                yield ("arrive", f"e_done{st}", 4)
                # one receive buffer (32 KB): free once the first CTA has read tile u - 1's
                if u >= 1 and "pair_rcv_free" not in drop:
                    if not (yield ("wait", "rcv_free0", u - 1)):
                        break
                yield ("write", "peer:rcv0")
                yield ("arrive", "peer:rcv_full0")
                yield ("arrive", f"stg_free{st}")
                continue
            if rank == 0:
                if "pair_rcv_full" not in drop:
                    if not (yield ("wait", "rcv_full0", u)):
                        break
                yield ("read", "rcv0")
                yield ("arrive", "peer:rcv_free0")
            if full_tile(u):
                yield ("write", f"hs{st}")
            yield ("arrive", f"e_done{st}", 4)
            if full_tile(u):
                yield ("write", f"hs{st}")
                yield ("store", (f"hs{st}",))
                if "y_store_wait" not in drop:
                    yield ("store_wait",)
                stored = True
            yield ("arrive", f"stg_free{st}")
        if stored:
            yield ("store_wait",)

    def e2_role():  # "E2": two-phase conversion in the E warps, then the fp32 state
        if nt == 0:
            return
        yield ("write", "hs0")
        yield ("arrive", "hs_ready0", 8)

        def convert_x(k):
            if not (yield ("wait", f"scan_done{k & 3}", k >> 2)) or not (yield ("wait", f"full{k & 1}", k >> 1)):
                return False
            yield ("read", f"ring{k & 3}")
            yield ("arrive", f"scan_free{k & 3}", 8)
            yield ("read", f"x{k & 1}")
            yield ("write", f"x{k & 1}")
            return True

        def write_wx(k):
            yield ("read", f"x{k & 1}")
            yield ("write", "wx")
            yield ("arrive", f"x_ready{k & 1}", 8)

        if not (yield from convert_x(0)):
            return
        yield from write_wx(0)
        for t in range(nt):
            if t + 1 < nt and not (yield from convert_x(t + 1)):
                break
            if not (yield ("wait", f"s_done{t & 1}", t >> 1)):
                break
            if t >= 1 and t + 1 < nt and "e_stg_free" not in drop:
                if not (yield ("wait", f"stg_free{(t + 1) & 1}", (t - 1) >> 1)):
                    break
            yield ("read", "tSt")
            yield ("arrive", f"st_free{t & 1}", 8)
            if t + 1 < nt:
                yield from write_wx(t + 1)
                yield ("write", f"hs{(t + 1) & 1}")
                yield ("arrive", f"hs_ready{(t + 1) & 1}", 8)

    def e_role():   # x operands and the fp32 state
        if nt > 0:
            yield ("write", "hs0")
            yield ("arrive", "hs_ready0", 8)
        for k in range(nt + 1):
            if k >= 1:
                u = k - 1
                if not (yield ("wait", f"s_done{u & 1}", u >> 1)):
                    break
                if 2 <= k < nt and "e_stg_free" not in drop:
                    if not (yield ("wait", f"stg_free{k & 1}", (k - 2) >> 1)):
                        break
                if conv != "E":
                    # 2^cs_last of tile u from the ring (ordered after the decay scan through
                    # x_ready -> s_done); the slot is released here
                    yield ("read", f"ring{u & 3}")
                    yield ("arrive", f"scan_free{u & 3}", 8)
                yield ("read", "tSt")
                if conv != "E":
                    yield ("arrive", f"st_free{u & 1}", 8)
                if k < nt:
                    yield ("write", f"hs{k & 1}")
                    yield ("arrive", f"hs_ready{k & 1}", 8)
            if k < nt and conv == "E":
                if not (yield from convert(k, 8)):
                    break

    roles = [("W19", w19()), ("W16", w16()), ("W18", w18()), ("W17", w17()), ("P", p_role()),
             ("Y", y_role()), ("E", e2_role() if conv == "E2" else e_role())]
    if y_issuer:
        roles.append(("W24", w24()))
    for name, gen in roles:
        m.role(pre + name, _prefixed(gen, pre, peer) if pair else gen)
    return m


def build_scan3_pair(nt: int, partial: bool = False, drop: frozenset = frozenset(), zero_b: str = "",
                     conv: str = "E") -> Machine:
    """The d_state 256 candidate: a cluster of two CTAs, each running the k_tc_scan3 roles on
    one half of the state rows (B and C halves), with one shared-memory stage for C.  The
    second CTA's epilogue writes its fp32 Y partial into the first CTA's receive buffer (one,
    32 KB: what the single C stage frees) and arrives on its rcv_full; the first CTA's epilogue
    adds it, stores y and arrives on the second CTA's rcv_free.  Both CTAs leave together (a
    cluster barrier)."""
    m = Machine()
    build_scan3(nt, partial, drop, zero_b, conv, m=m, rank=0)
    build_scan3(nt, partial, drop, zero_b, conv, m=m, rank=1)
    return m


# The first-generation kernel (k_tc_scan<N>, N = 256): state accumulated in TMEM.
# One B/C stage, loaded as four 64-column boxes with a barrier each (its reload
# waits for the tile's C B^T, C h_prev and B^T (w o x)); one Yd buffer (its S x
# waits for the previous epilogue), Yo per tile parity.  Three MMA-issuing
# threads: W16 (C B^T), W17 (C h_prev, then S x) and W18 (B^T (w o x), state
# rows of boxes 0-1, then 2-3); sc_done completes once W17 and W18 have both
# committed.  On a partial last tile, W18 waits for P to zero the B rows past
# the sequence end (b_zeroed, used once).  `fin`: the MMA-issuing threads drain
# their tensor-core work before the CTA exits.

BOXES = 4


def build_scan1(nt: int, partial: bool = False, drop: frozenset = frozenset(), fin: bool = True) -> Machine:
    m = Machine()
    for i in range(2):
        m.barrier(f"xfull{i}", 1)
        m.barrier(f"scan_done{i}", 8)
        m.barrier(f"e_done{i}", 8)
        m.barrier(f"x_ready{i}", 8)
        m.barrier(f"yd_par{i}", 1)
    for k in range(BOXES):
        m.barrier(f"bcfull{k}", 1)
    for i in range(3):
        m.barrier(f"fin{i}", 1)
    for name, count in (("cb_done", 1), ("s_ready", 8), ("sc_done", 2), ("b_zeroed", 8)):
        m.barrier(name, count)
    last_partial = lambda t: partial and t == nt - 1
    b_all = tuple(f"b{k}" for k in range(BOXES))

    def w16():      # TMA and C B^T
        if nt == 0:
            return
        issued = {"x": 0, "bc": 0}

        def load_x(t):
            yield ("arrive_tx", f"xfull{t & 1}", 1)
            yield ("tma_load", f"xfull{t & 1}", f"x{t & 1}")
            issued["x"] += 1

        def load_bc():
            for k in range(BOXES):
                yield ("arrive_tx", f"bcfull{k}", 2)
                yield ("tma_load", f"bcfull{k}", f"b{k}")
                yield ("tma_load", f"bcfull{k}", f"c{k}")
            issued["bc"] += 1

        yield from load_x(0)
        yield from load_bc()
        if nt > 1:
            yield from load_x(1)
        ok = True
        for t in range(nt):
            if t > 0 and "w16_s_ready" not in drop:
                if not (ok := (yield ("wait", "s_ready", t - 1))):
                    break
            for k in range(BOXES):
                if not (ok := (yield ("wait", f"bcfull{k}", t))):
                    break
                yield ("mma", (f"c{k}", f"b{k}"), ("tCB",))
            if not ok:
                break
            yield ("commit", "cb_done")
            if t >= 1 and t + 1 < nt:
                if "w16_yd_par" not in drop:
                    if not (ok := (yield ("wait", f"yd_par{(t - 1) & 1}", (t - 1) >> 1))):
                        break
                yield from load_x(t + 1)
            if t + 1 < nt:
                if "w16_cb_done" not in drop:
                    if not (ok := (yield ("wait", "cb_done", t))):
                        break
                if "w16_sc_done" not in drop:
                    if not (ok := (yield ("wait", "sc_done", t))):
                        break
                yield from load_bc()
        if not ok:
            for t in range(issued["x"]):
                yield ("bwait", f"xfull{t & 1}", t >> 1)
            for t in range(issued["bc"]):
                for k in range(BOXES):
                    yield ("bwait", f"bcfull{k}", t)
        if fin:
            yield ("commit", "fin0")
            yield ("bwait", "fin0", 0)

    def w17():      # C h_prev, box by box, then S x
        ok = True
        for t in range(nt):
            st = t & 1
            if not (ok := (yield ("wait", f"x_ready{st}", t >> 1))):
                break
            for k in range(BOXES):
                if "w17_bcfull" not in drop:
                    if not (ok := (yield ("wait", f"bcfull{k}", t))):
                        break
                yield ("mma", (f"c{k}", "hs"), (f"tYo{st}",))
            if not ok:
                break
            yield ("commit", "sc_done")
            if "w17_s_ready" not in drop:
                if not (ok := (yield ("wait", "s_ready", t))):
                    break
            if t > 0 and "w17_e_done" not in drop:
                if not (ok := (yield ("wait", f"e_done{(t - 1) & 1}", (t - 1) >> 1))):
                    break
            yield ("mma", ("tS", f"x{st}"), ("tYd",))
            yield ("commit", f"yd_par{st}")
        if fin and nt > 0:
            yield ("commit", "fin1")
            yield ("bwait", "fin1", 0)

    def w18():      # H += B^T (w o x), state rows of boxes 0-1, then 2-3
        ok = True
        for t in range(nt):
            if not (ok := (yield ("wait", f"x_ready{t & 1}", t >> 1))):
                break
            if last_partial(t) and "w18_b_zeroed" not in drop:
                if not (ok := (yield ("wait", "b_zeroed", 0))):
                    break
            for mb in range(BOXES // 2):
                for k in (2 * mb, 2 * mb + 1):
                    if "w18_bcfull" not in drop:
                        if not (ok := (yield ("wait", f"bcfull{k}", t))):
                            break
                if not ok:
                    break
                yield ("mma", (f"b{2 * mb}", f"b{2 * mb + 1}", "wx", f"tH{mb}"), (f"tH{mb}",))
            if not ok:
                break
            yield ("commit", "sc_done")
        if fin and nt > 0:
            yield ("commit", "fin2")
            yield ("bwait", "fin2", 0)

    def p_role():
        yield ("write", "tS")
        for t in range(nt):
            buf = t & 1
            if t >= 2 and "p_e_done" not in drop:
                if not (yield ("wait", f"e_done{buf}", (t - 2) >> 1)):
                    break
            yield ("write", f"ring{buf}")
            yield ("arrive", f"scan_done{buf}", 8)
            if not (yield ("wait", "cb_done", t)):
                break
            if last_partial(t):
                yield ("write", *b_all)             # rows past the sequence end zeroed
                yield ("arrive", "b_zeroed", 8)
            if t > 0 and "p_yd_par" not in drop:
                if not (yield ("wait", f"yd_par{(t - 1) & 1}", (t - 1) >> 1)):
                    break
            yield ("read", "tCB", f"ring{buf}")
            yield ("write", "tS")
            yield ("arrive", "s_ready", 8)

    def e_role():
        def prepare(u):
            st = u & 1
            if not (yield ("wait", f"scan_done{st}", u >> 1)):
                return False
            yield ("read", f"ring{st}")
            if u > 0:
                yield ("read", "tH0", "tH1")
            yield ("write", "hs", "tH0", "tH1")
            if not (yield ("wait", f"xfull{st}", u >> 1)):
                return False
            yield ("read", f"x{st}")
            yield ("write", f"x{st}", "wx")
            yield ("arrive", f"x_ready{st}", 8)
            return True

        ok = True
        for k in range(nt + 1):
            # sc_done of tile k - 1: the state entering tile k is complete, hs and w o x are
            # free, and C h_prev of tile k - 1 (read by its epilogue) is done
            if k > 0 and not (k == nt and "e_last_sc_done" in drop) and not (k < nt and "e_sc_done" in drop):
                if not (ok := (yield ("wait", "sc_done", k - 1))):
                    break
            if k < nt and not (ok := (yield from prepare(k))):
                break
            if k == 0:
                continue
            t = k - 1
            st = t & 1
            if not (ok := (yield ("wait", f"yd_par{st}", t >> 1))):
                break
            yield ("read", f"ring{st}", "tYd", f"tYo{st}")
            yield ("arrive", f"e_done{st}", 8)
        if nt > 0 and ok:
            yield ("read", "tH0", "tH1")               # the final state

    for name, gen in (("W16", w16()), ("W17", w17()), ("W18", w18()), ("P", p_role()), ("E", e_role())):
        m.role(name, gen)
    return m


def check(build, schedules: int, seed: int, faults: bool = False, **kw) -> None:
    """Runs `schedules` random schedules of the model `build(**kw)`; raises ProtocolError on the first
    race, deadlock, aliasing or exit with work in flight.  With `faults`, each schedule also times
    out one waiting role at a random step (the timeout path: only deadlock and exit with work in
    flight are checked from there on)."""
    rng = random.Random(seed)
    for _ in range(schedules):
        m = build(**kw)
        m.run(rng, fault_at=rng.randrange(0, 40 * (kw.get("nt", 1) + 1)) if faults else None)


# ---------------------------------------------------------------------------
# Leader waits inside a role.  A role of several warps waits as one: the leader
# polls the mbarrier, writes the result to a flag in shared memory, all warps
# meet at a named barrier (bar.sync, no timeout) and each reads the flag.  With
# one flag the leader's next write can land before a slow warp has read the
# previous result; warps of one role then disagree, and a warp that leaves
# while the others go on to the next bar.sync leaves them waiting forever.
# Alternating between two flags closes this: the leader writes a slot again
# only after the next bar.sync, which every warp passes after its read.

def role_leader_waits(nwarps: int, results, slots: int, rng: random.Random) -> str | None:
    """Runs one random schedule of `nwarps` warps through consecutive leader waits whose
    outcomes are `results` (False = the leader's wait gave up); returns None, or a description
    of a warp that read another wait's result or of a hang at a named barrier."""
    flag = [None] * slots
    arrived, gen = 0, 0
    pc = [("write" if w == 0 else "sync", 0) for w in range(nwarps)]   # (next action, call index)
    waiting_gen = [None] * nwarps
    done = [False] * nwarps
    weight = [10 ** rng.uniform(-3, 0) for _ in range(nwarps)]
    ncalls = len(results)
    while not all(done):
        runnable = []
        for w in range(nwarps):
            if done[w]:
                continue
            act, i = pc[w]
            if act == "blocked" and gen == waiting_gen[w]:
                continue                                   # still parked at the named barrier
            runnable.append(w)
        if not runnable:
            return "hang: warps parked at a named barrier that a departed warp never reaches"
        w = rng.choices(runnable, [weight[v] for v in runnable])[0]
        act, i = pc[w]
        if act == "write":                                 # leader: the wait's result
            flag[i % slots] = (i, results[i])
            pc[w] = ("sync", i)
        elif act == "sync":
            arrived += 1
            if arrived == nwarps:                          # last arrival releases the barrier
                arrived, gen = 0, gen + 1
                pc[w] = ("read", i)
            else:
                waiting_gen[w] = gen
                pc[w] = ("blocked", i)
        elif act == "blocked":                             # released
            pc[w] = ("read", i)
        elif act == "read":
            call, value = flag[i % slots]
            if call != i:
                return f"warp {w} read the result of wait {call} for wait {i}"
            if not value or i + 1 == ncalls:
                done[w] = True                             # leaves the role's loop
            else:
                pc[w] = ("write" if w == 0 else "sync", i + 1)
    return None
