"""A discrete-event model of the barrier protocol of the fused MLP GEMM (gemm_swiglu_quant_kernel in
csrc/svdq_fused.cuh), checked on the host.

Every role of both CTAs of a pair (producer, MMA issuer, scale-factor writers, epilogue warps)
replays, in the kernel's order, its barrier waits, arrivals and multicast commits. Barriers follow
mbarrier semantics: an arrival count per phase, waits on phase parity. Copies landing and MMA
commits completing are delivered late and in random order. At every use of a shared resource the
model asserts that its previous user is done:
  * a ring stage is refilled only after the MMAs that read it completed;
  * a slot's MMAs are issued only once both CTAs' copies of it have landed;
  * the accumulator is overwritten only after every epilogue warp has read the previous tile;
  * the h tile is rewritten only after the previous tile's U' MMAs read it;
  * a tile's L1s' slice travels in a ring slot of its own, loaded after the next tile's K steps:
    its U' MMAs are issued only once both CTAs' halves of it have landed, and release the slot;
  * a unit's first U' MMA (accumulate = 0) comes only after the previous unit's U' was drained.
Over many schedules and unit layouts the model must finish without a deadlock or stray arrivals,
and every wait must pass on exactly the completion it means (a parity wait a phase early passes too
soon; two phases late it blocks forever on hardware). Removing any one wait must make it fail.

The model transcribes the kernel's roles as barrier traffic only; it does not run the kernel."""
import random

import pytest

SF_BUFS = 4
KERNEL_STAGES = 5   # the fused kernel's ring depth (kFusedStages)

# Waits whose removal must break the protocol. Two of the kernel's waits are implied by others:
#  * issuer.u_free: a unit's first U' MMA waits on h_full, and the draining warps arrive on h_full
#    only after their drain (the kernel keeps the wait as a cheap safeguard);
#  * sf.release, while the ring has no more stages than scale buffers: a writer cannot see the
#    data of the slot SF_BUFS ahead before this slot is consumed. With a deeper ring (the NVFP4
#    GEMM runs 5 stages) it is needed, which test_every_wait_is_needed checks at 6 stages.
WAITS = ["producer.empty", "issuer.acce", "issuer.sf_full", "issuer.slice_sf_full", "issuer.h_full",
         "sf.full", "sf.release", "epi.accf", "epi.u_done", "epi.h_empty"]


class Barrier:
    def __init__(self, name, count):
        self.name, self.count, self.pending, self.completed = name, count, count, 0

    def arrive(self, n=1):
        self.pending -= n
        assert self.pending >= 0, f"{self.name}: more arrivals than its count in one phase"
        if self.pending == 0:
            self.completed += 1
            self.pending = self.count


def run_model(units, r, k_iters, seed, skip=(), stages=KERNEL_STAGES):
    """units: tile counts of the units one CTA pair sweeps, in order. skip: waits to leave out."""
    STAGES = stages
    rng = random.Random(seed)
    slots = (r + 31) // 32 + k_iters
    B = {}

    def bar(name, count):
        B[name] = Barrier(name, count)

    for c in (0, 1):
        for s in range(STAGES):
            bar(f"full{c}.{s}", 1)
            bar(f"empty{c}.{s}", 1)
        bar(f"accf{c}", 1)
        bar(f"h_empty{c}", 1)
        bar(f"u_done{c}", 1)
    bar("acce", 16)                     # 8 epilogue warps x 2 CTAs
    for b in range(SF_BUFS):
        bar(f"sf_full{b}", 8)           # 4 writer warps x 2 CTAs
    bar("h_full", 16)
    bar("u_free", 8)                    # 4 draining warps x 2 CTAs
    done = lambda name: B[name].completed  # noqa: E731

    in_flight = []                      # copies landing / MMA commits completing

    def later(name):
        in_flight.append(name)

    def wait(tag, name, index):
        """Wait, as the kernel does, by parity for completion #index of `name` (index -1: the
        first use, which a fresh barrier passes at once)."""
        if tag in skip:
            return
        while (B[name].completed & 1) == (index & 1):
            yield name
        assert B[name].completed == index + 1, \
            f"{name}: wait for completion #{index} passed at completed = {B[name].completed}"

    tiles = [(t == 0, t == n - 1) for n in units for t in range(n)]

    # the ring slots of one pair in order: per tile its low-rank and K-step slots, then (from the
    # second tile on) the previous tile's slice slot; after the last tile, its slice slot
    order = []
    for t in range(len(tiles)):
        order += ["data"] * slots + (["slice"] if t > 0 else [])
    if tiles:
        order.append("slice")

    def producer(c):
        stage = 0
        uses = [0] * STAGES
        for _ in order:
            yield from wait("producer.empty", f"empty{c}.{stage}", uses[stage] - 1)
            assert done(f"empty{c}.{stage}") >= uses[stage], "ring stage refilled while its MMAs read it"
            uses[stage] += 1
            later(f"full{c}.{stage}")
            stage = (stage + 1) % STAGES

    def issuer():
        stage, sfb, useq, g = 0, 0, 0, 0
        sf_uses = [0] * SF_BUFS
        pend = None

        def issue_u(t, first, last):
            nonlocal useq, stage, sfb, g
            yield from wait("issuer.h_full", "h_full", t)
            if first and useq > 0:
                yield from wait("issuer.u_free", "u_free", useq - 1)
            yield from wait("issuer.slice_sf_full", f"sf_full{sfb}", sf_uses[sfb])
            sf_uses[sfb] += 1
            for c in (0, 1):
                assert done(f"full{c}.{stage}") >= g // STAGES + 1, "U' MMA before a CTA's slice landed"
            assert done("h_full") >= t + 1, "U' MMA before both h tiles were written"
            if first:
                assert done("u_free") >= useq, "U' overwritten before the previous unit was drained"
            for c in (0, 1):
                later(f"empty{c}.{stage}")
                later(f"h_empty{c}")
                if last:
                    later(f"u_done{c}")
            stage = (stage + 1) % STAGES
            sfb = (sfb + 1) % SF_BUFS
            g += 1
            if last:
                useq += 1

        for tseq, (first, last) in enumerate(tiles):
            yield from wait("issuer.acce", "acce", tseq - 1)
            assert done("acce") >= tseq, "accumulator overwritten before the epilogue read it"
            for _ in range(slots):
                yield from wait("issuer.sf_full", f"sf_full{sfb}", sf_uses[sfb])
                sf_uses[sfb] += 1
                for c in (0, 1):
                    assert done(f"full{c}.{stage}") >= g // STAGES + 1, "MMA before a CTA's copy landed"
                for c in (0, 1):
                    later(f"empty{c}.{stage}")
                stage = (stage + 1) % STAGES
                sfb = (sfb + 1) % SF_BUFS
                g += 1
            if pend is not None:
                yield from issue_u(*pend)
            for c in (0, 1):
                later(f"accf{c}")
            pend = (tseq, first, last)
        if pend is not None:
            yield from issue_u(*pend)

    def sf_writers(c):
        # a CTA's 4 writer warps move in step; together they arrive 4 times per slot
        full_uses = [0] * STAGES
        released = [0] * STAGES
        stage, sfb, n = 0, 0, 0
        for _ in order:
            yield from wait("sf.full", f"full{c}.{stage}", full_uses[stage])
            full_uses[stage] += 1
            if n >= SF_BUFS:
                ps = (stage - SF_BUFS) % STAGES               # the slot SF_BUFS back
                yield from wait("sf.release", f"empty{c}.{ps}", released[ps])
                released[ps] += 1
            B[f"sf_full{sfb}"].arrive(4)
            n += 1
            stage = (stage + 1) % STAGES
            sfb = (sfb + 1) % SF_BUFS

    def epilogue(c, drains):
        useq = 0

        def drain(u):
            yield from wait("epi.u_done", f"u_done{c}", u)
            assert done(f"u_done{c}") >= u + 1, "U' drained before its MMAs completed"
            B["u_free"].arrive()

        for tseq, (first, last) in enumerate(tiles):
            yield from wait("epi.accf", f"accf{c}", tseq)
            assert done(f"accf{c}") >= tseq + 1, "accumulator read before its MMAs completed"
            if first and useq > 0 and drains:
                yield from drain(useq - 1)
            if tseq > 0:
                yield from wait("epi.h_empty", f"h_empty{c}", tseq - 1)
            assert done(f"h_empty{c}") >= tseq, "h tile rewritten while U' MMAs read it"
            B["acce"].arrive()
            B["h_full"].arrive()
            if last:
                useq += 1
        if useq > 0 and drains:
            yield from drain(useq - 1)

    live = {"issuer": issuer()}
    for c in (0, 1):
        live[f"producer{c}"] = producer(c)
        live[f"sf{c}"] = sf_writers(c)
        for w in range(8):
            live[f"epi{c}.{w}"] = epilogue(c, drains=w < 4)   # warps 2..5 (h = 0) drain U'

    for _ in range(1_000_000):
        if not live:
            break
        waiting = {}
        for k in rng.sample(sorted(live), len(live)):
            try:
                waiting[k] = next(live[k])
            except StopIteration:
                del live[k]
        if live and not in_flight and all(waiting.get(k) is not None for k in live):
            still = {}
            for k in list(live):
                try:
                    still[k] = next(live[k])
                except StopIteration:
                    del live[k]
            if live and not in_flight and all(v is not None for v in still.values()):
                raise AssertionError(f"deadlock: {still}")
        rng.shuffle(in_flight)
        for _ in range(rng.randint(0, len(in_flight))):
            B[in_flight.pop()].arrive()
    assert not live, "model did not finish"
    while in_flight:
        B[in_flight.pop()].arrive()
    for name, b in B.items():
        assert b.pending == b.count, f"{name}: {b.count - b.pending} stray arrivals at the end"
    return True


LAYOUTS = [[1], [3], [1, 1, 1], [2, 1], [1, 2, 3], [5, 5], [4, 1, 2, 1], [24]]
SHAPES = [(32, 2), (64, 1), (0, 3), (16, 12)]


@pytest.mark.parametrize("units", LAYOUTS)
@pytest.mark.parametrize("r,k_iters", SHAPES)
def test_fused_protocol_model(units, r, k_iters):
    for seed in range(5):
        assert run_model(units, r, k_iters, seed)


@pytest.mark.parametrize("stages", [KERNEL_STAGES, 6])
def test_deeper_ring(stages):
    for units in ([2, 3], [24]):
        for r, k_iters in SHAPES:
            for seed in range(3):
                assert run_model(units, r, k_iters, seed, stages=stages)


@pytest.mark.parametrize("skipped", WAITS)
def test_every_wait_is_needed(skipped):
    """Without any one of its waits the protocol fails somewhere: a resource reused too early, an
    arrival landing in the wrong phase, a wait passing on the wrong completion, or a deadlock."""
    stages = 6 if skipped == "sf.release" else KERNEL_STAGES
    for units in ([2, 3], [1, 1, 1], [5, 5], [24]):
        for r, k_iters in SHAPES:
            for seed in range(20):
                try:
                    run_model(units, r, k_iters, seed, skip={skipped}, stages=stages)
                except AssertionError:
                    return
    pytest.fail(f"removing the wait {skipped} went unnoticed")


def test_u_free_is_implied_by_h_full():
    """The kernel's u_free wait never decides anything (see WAITS): leaving it out changes no run."""
    for units in ([2, 3], [1, 1, 1], [5, 5]):
        for r, k_iters in SHAPES:
            for seed in range(5):
                assert run_model(units, r, k_iters, seed, skip={"issuer.u_free"})
