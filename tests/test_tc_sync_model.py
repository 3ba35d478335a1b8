"""The role hand-off protocol of the tensor-core scan kernels, model-checked on the CPU.

``tests/tc_sync_model.py`` restates, per role and tile, the mbarrier waits, arrivals,
buffer accesses and async copies / MMAs of ``k_tc_scan3`` (d_state 128) and of the
first-generation ``k_tc_scan<N>`` (d_state 256, and its 128 configuration), and runs
them under random schedules with vector-clock race detection.  The tests check that
the protocol has no race, deadlock or parity aliasing for 0 .. 9 tiles (full and
ragged last tile), and that removing any wait the protocol needs is caught.
"""
import random

import pytest

from tests.tc_sync_model import Barrier, Machine, ProtocolError, build_scan1, build_scan3, check

TILES = (0, 1, 2, 3, 4, 5, 6, 9)


# ---- the checker itself -------------------------------------------------------------


def test_barrier_parity_and_transaction_rules():
    b = Barrier("b", 2)
    assert b.try_wait(0) == (False, None)
    b.arrive({"a": 1}, tx=3)
    b.arrive({"c": 1})
    assert not b.try_wait(0)[0]             # arrivals done, bytes outstanding
    b.complete_tx({"tma": 1}, 3)
    ok, vc = b.try_wait(0)
    assert ok and vc == {"a": 1, "c": 1, "tma": 1}
    b.arrive({}, weight=2)                  # phase 1 completes: a waiter for phase 0 now sees parity 0 again
    with pytest.raises(ProtocolError, match="two phases past"):
        b.try_wait(0)
    b2 = Barrier("b2", 1)
    b2.arrive({})
    with pytest.raises(ProtocolError, match="aliasing"):
        b2.try_wait(2)                      # a waiter two phases ahead would pass on phase 0
    with pytest.raises(ProtocolError, match="more arrivals"):
        Barrier("b3", 1).arrive({}, weight=2)


def _two_roles(ordered):
    m = Machine()
    m.barrier("ready", 1)

    def producer():
        yield ("write", "buf")
        yield ("arrive", "ready")

    def consumer():
        if ordered:
            yield ("wait", "ready", 0)
        yield ("read", "buf")

    m.role("prod", producer())
    m.role("cons", consumer())
    return m


def test_race_detector_needs_the_barrier_and_accepts_it():
    found = False
    rng = random.Random(0)
    for _ in range(50):
        _two_roles(True).run(rng)
        try:
            _two_roles(False).run(rng)
        except ProtocolError as e:
            found = found or "race on buf" in str(e)
    assert found


def test_async_mma_is_ordered_only_through_its_commit():
    def build(wait_commit):
        m = Machine()
        m.barrier("done", 1)

        def issuer():
            yield ("mma", ("a",), ("acc",))
            yield ("commit", "done")

        def reader():
            if wait_commit:
                yield ("wait", "done", 0)
            yield ("read", "acc")

        m.role("W", issuer())
        m.role("R", reader())
        return m

    rng = random.Random(1)
    for _ in range(50):
        build(True).run(rng)
    with pytest.raises(ProtocolError):
        for _ in range(200):
            build(False).run(rng)


def test_exit_with_work_in_flight_is_reported():
    m = Machine()

    def issuer():
        yield ("mma", (), ("acc",))           # issued, never committed and waited for

    m.role("W", issuer())
    with pytest.raises(ProtocolError, match="in flight"):
        m.run(random.Random(0))


# ---- the kernels ----------------------------------------------------------------------


@pytest.mark.parametrize("partial", [False, True])
def test_scan3_protocol_has_no_race_deadlock_or_aliasing(partial):
    for nt in TILES:
        check(build_scan3, 25, seed=100 + nt, nt=nt, partial=partial)


@pytest.mark.parametrize("partial", [False, True])
def test_scan1_protocol_has_no_race_deadlock_or_aliasing(partial):
    for nt in TILES:
        check(build_scan1, 25, seed=200 + nt, nt=nt, partial=partial)


def _caught(build, drop, **kw):
    for nt in (1, 3, 5, 8):
        for partial in (False, True):
            try:
                check(build, 40, seed=nt, nt=nt, partial=partial, drop=frozenset([drop]), **kw)
            except ProtocolError as e:
                return str(e)
    return None


NEEDED = [
    (build_scan3, {}, "w19_scan_free", "ring"),
    (build_scan3, {}, "w16_y_full", "x0"),
    (build_scan3, {}, "w18_cb_free", "tCB"),
    (build_scan3, {}, "w17_s_ready", "tS"),
    (build_scan3, {}, "p_y_full", "tS"),
    (build_scan3, {}, "y_store_wait", "hs"),
    (build_scan3, {}, "e_stg_free", "hs"),
    (build_scan1, {}, "w16_s_ready", "tCB"),
    (build_scan1, {}, "w16_yd_par", "x"),
    (build_scan1, {}, "w16_sc_done", ""),
    (build_scan1, {}, "w16_cb_done", ""),
    (build_scan1, {}, "w17_bcfull", "c"),
    (build_scan1, {}, "w18_bcfull", "b"),
    (build_scan1, {}, "w18_b_zeroed", "b"),
    (build_scan1, {}, "w17_s_ready", "tS"),
    (build_scan1, {}, "w17_e_done", "tYd"),
    (build_scan1, {}, "p_e_done", "ring"),
    (build_scan1, {}, "p_yd_par", "tS"),
    (build_scan1, {}, "e_sc_done", ""),
    (build_scan1, {}, "e_last_sc_done", "tH"),
]


@pytest.mark.parametrize("build,kw,drop,buf", NEEDED, ids=[f"{b.__name__}-{d}" for b, kw, d, _ in NEEDED])
def test_removing_a_needed_wait_is_caught(build, kw, drop, buf):
    msg = _caught(build, drop, **kw)
    assert msg is not None and "race on " + buf in msg, msg


def test_waits_implied_by_other_waits():
    """Waits the kernels keep although another wait already implies them:
    k_tc_scan3's W18 y_full wait (its full-barrier wait follows W16's y_full wait), W17's
    e_done wait (hs_ready follows E's stg_free wait, which follows Y's read of the Y buffer).
    The tensor-core drains before exit (fin) matter only on the timeout path (tested below)."""
    for build, kw, drop in ((build_scan3, {}, "w18_y_full"), (build_scan3, {}, "w17_e_done"),
                            (build_scan3, {}, "w17_fin"), (build_scan3, {}, "w18_fin")):
        assert _caught(build, drop, **kw) is None, drop


# ---- the timeout path -------------------------------------------------------------------
# A bounded wait that gives up sets the CTA's abort flag; every later wait gives up at
# once, each role leaves its loop, and before the CTA frees TMEM and exits every TMA copy
# and tcgen05 operation it issued must have completed.


def _faults(build, drop=frozenset(), **kw):
    try:
        for nt in (1, 2, 3, 5, 7):
            for partial in (False, True):
                check(build, 60, seed=300 + nt, faults=True, nt=nt, partial=partial, drop=drop, **kw)
    except ProtocolError as e:
        return str(e)
    return None


def test_scan3_timeout_path_exits_with_nothing_in_flight():
    assert _faults(build_scan3) is None


@pytest.mark.parametrize("drain", ["w16_drain", "w17_fin", "w18_fin"])
def test_scan3_needs_each_of_its_drains(drain):
    assert "in flight" in (_faults(build_scan3, frozenset([drain])) or "")


def test_scan1_timeout_path_needs_its_mma_drains():
    """The first-generation kernel's MMA-issuing threads drain their tensor-core work before
    exit; without that, a timeout can leave MMAs writing TMEM after it is freed."""
    assert _faults(build_scan1) is None
    assert "in flight" in (_faults(build_scan1, fin=False) or "")


def test_planned_zeroing_of_b_rows_past_a_sequence_end():
    """k_tc_scan3 does not yet zero the B rows past a sequence's end in its partial last tile
    (they feed B^T (w o x) against exact zeros, so only a non-finite B of the next sequence
    matters).  Of two ways to add it, zeroing in the P warps after C B^T has read B, with W17
    waiting for c_scaled before B^T (w o x) on that tile, is race-free, also on the timeout path;
    zeroing in the E warps before x_ready races with W18's C B^T read."""
    for nt in (1, 2, 3, 5, 8):
        check(build_scan3, 40, seed=400 + nt, nt=nt, partial=True, zero_b="p")
        check(build_scan3, 20, seed=500 + nt, nt=nt, partial=True, zero_b="p", faults=True)
    with pytest.raises(ProtocolError, match="race on b"):
        for nt in (1, 2, 3, 5, 8):
            check(build_scan3, 40, seed=600 + nt, nt=nt, partial=True, zero_b="e")


def test_candidate_conversion_in_the_epilogue_warps():
    """A candidate restructuring of k_tc_scan3 (not built yet): the epilogue warps convert x of
    tile t + 1 as soon as B^T (w o x) of tile t has completed, and the E warps only update the
    state.  The single TMEM buffer of the tile's own state term then needs its own release: E
    arrives at st_free right after loading s, and W17 waits for it before the next B^T (w o x).
    With that the protocol is clean, also on the timeout path; without it the next MMA can
    overwrite s while E is still reading it."""
    for nt in (0, 1, 2, 3, 5, 9):
        for partial in (False, True):
            check(build_scan3, 30, seed=700 + nt, nt=nt, partial=partial, conv="Y")
            check(build_scan3, 15, seed=800 + nt, nt=nt, partial=partial, conv="Y", faults=True)
    with pytest.raises(ProtocolError, match="race on tSt"):
        for nt in (2, 3, 5, 9):
            check(build_scan3, 40, seed=900 + nt, nt=nt, conv="Y", drop=frozenset(["w17_st_free"]))
    # together with the zeroing of B rows past a sequence end, and in the two-phase form (x
    # converted in place as soon as it lands, w o x written after B^T (w o x) of the tile before)
    for conv in ("Y", "Y2"):
        for nt in (1, 2, 5):
            check(build_scan3, 30, seed=950 + nt, nt=nt, partial=True, conv=conv, zero_b="p")
            check(build_scan3, 15, seed=960 + nt, nt=nt, partial=True, conv=conv, zero_b="p", faults=True)
    for nt in (0, 3, 9):
        check(build_scan3, 30, seed=970 + nt, nt=nt, conv="Y2")
    # the lean form of the draft: without the two waits that other waits imply (W18's y_full,
    # W17's e_done, hence no e_done barrier at all)
    lean = frozenset(["w17_e_done", "w18_y_full"])
    for nt in (1, 2, 5, 9):
        check(build_scan3, 30, seed=980 + nt, nt=nt, partial=True, conv="Y2", zero_b="p", drop=lean)
        check(build_scan3, 15, seed=990 + nt, nt=nt, partial=True, conv="Y2", zero_b="p", drop=lean, faults=True)


def test_role_leader_flag_needs_two_slots():
    """One flag per role lets a slow warp read the leader's next result (and, when that wait
    gave up, leave while the others park at the next named barrier); two alternating flags
    never do, whatever the schedule."""
    from tests.tc_sync_model import role_leader_waits
    rng = random.Random(5)
    results = [True] * 5 + [False]
    one = [role_leader_waits(8, results, 1, rng) for _ in range(400)]
    assert any(r is not None for r in one)
    for _ in range(400):
        assert role_leader_waits(8, results, 2, rng) is None
        assert role_leader_waits(4, [True] * 7, 2, rng) is None


def test_dstate_256_pair_candidate():
    """The d_state 256 candidate: two CTAs of a cluster run the k_tc_scan3 roles on the two
    halves of the state rows, C has one shared-memory stage (reloaded once its copy to TMEM has
    completed), and the second CTA's fp32 Y partial travels to the first CTA through distributed
    shared memory (one receive buffer, rcv_full / rcv_free).  Clean, also on the timeout path and
    with the conversion and tail-zeroing candidates; each of its three new waits is needed."""
    from tests.tc_sync_model import build_scan3_pair
    for nt in (0, 1, 2, 3, 5, 9):
        for partial in (False, True):
            check(build_scan3_pair, 15, seed=1000 + nt, nt=nt, partial=partial)
            check(build_scan3_pair, 8, seed=1100 + nt, nt=nt, partial=partial, faults=True)
    for nt in (2, 5):
        check(build_scan3_pair, 15, seed=1200 + nt, nt=nt, partial=True, conv="Y2", zero_b="p")
    for drop, what in (("pair_rcv_full", r"a\.rcv"), ("pair_rcv_free", r"rcv"),
                       ("pair_c_stage", r"cfull|c0")):
        with pytest.raises(ProtocolError, match=what):
            for nt in (3, 5, 8):
                check(build_scan3_pair, 30, seed=1300 + nt, nt=nt, drop=frozenset([drop]))


def test_two_phase_conversion_in_the_e_warps():
    """The E warps convert x of tile t + 1 in place while B^T (w o x) of tile t runs; after it
    completes they load s, write w o x of tile t + 1 and the state entering it.  With the B rows
    past a sequence end zeroed by P and without the waits other waits imply, the protocol is
    clean, also on the timeout path.  Implied waits: W18's y_full and W17's e_done (as in the
    epilogue-warp forms), and here also W17's st_free: E loads s(t) before it writes w o x of
    tile t + 1, so x_ready(t + 1) already orders the next B^T (w o x) after that load.  The
    stg_free wait before the state copy (hs doubles as the y staging buffer) is needed."""
    lean = frozenset(["w17_e_done", "w18_y_full", "w17_st_free"])
    for nt in (0, 1, 2, 3, 5, 9):
        for partial in (False, True):
            check(build_scan3, 30, seed=1300 + nt, nt=nt, partial=partial, conv="E2", zero_b="p", drop=lean)
            check(build_scan3, 15, seed=1400 + nt, nt=nt, partial=partial, conv="E2", zero_b="p", drop=lean,
                  faults=True)
    with pytest.raises(ProtocolError):
        for nt in (3, 5, 9):
            check(build_scan3, 40, seed=1600 + nt, nt=nt, conv="E2", zero_b="p", drop=lean | {"e_stg_free"})


def test_kernel_form_with_a_separate_output_chain_issuer():
    """k_tc_scan3 as built: the two-phase conversion in the E warps, the B rows past a sequence
    end zeroed by P, and the output chain (C' h_prev, S x) on its own issuing warp (W24) beside
    W17's B^T (w o x), without the waits other waits imply.  Clean, also on the timeout path;
    W24's own waits for x_ready (S x reads the converted x), s_ready and its drain are each
    needed, and so is W16's wait for s_done before it reloads a stage: W24's y_full commit does
    not cover W17's B^T (w o x), which reads the stage's B."""
    lean = frozenset(["w17_e_done", "w18_y_full", "w17_st_free"])
    kw = dict(conv="E2", zero_b="p", y_issuer=True)
    for nt in (0, 1, 2, 3, 5, 9):
        for partial in (False, True):
            check(build_scan3, 30, seed=1700 + nt, nt=nt, partial=partial, drop=lean, **kw)
            check(build_scan3, 15, seed=1800 + nt, nt=nt, partial=partial, drop=lean, faults=True, **kw)
    with pytest.raises(ProtocolError, match="race on x"):
        for nt in (1, 2, 3):
            check(build_scan3, 40, seed=1900 + nt, nt=nt, drop=lean | {"w24_x_ready"}, **kw)
    with pytest.raises(ProtocolError, match="race on tS"):
        for nt in (2, 3, 5):
            check(build_scan3, 40, seed=2000 + nt, nt=nt, drop=lean | {"w17_s_ready"}, **kw)
    assert "in flight" in (_faults(build_scan3, drop=lean | {"w24_fin"}, **kw) or "")
    with pytest.raises(ProtocolError, match="race on b"):
        for nt in (3, 5, 9):
            check(build_scan3, 60, seed=2100 + nt, nt=nt, drop=lean | {"w16_s_done"}, **kw)
