"""A discrete-event model of the barrier protocol of the CTA-pair GEMM (pair_gemm_kernel in
csrc/svdq_gemm.cuh, for both formats: NVFP4 with its scale factors, and row-wise FP8 without),
checked on the host like test_fused_protocol_model.py: producer, MMA issuer, the four scale-factor
writer warps (NVFP4 only) and the eight epilogue warps of both CTAs replay their barrier traffic in
the kernel's order, with copies and MMA completions landing late and in random order.

Protocol per ring slot: both CTAs' A / B (or low-rank) copies complete on the even CTA's full
barrier, whose phase also needs the even producer's arrive (it expects both CTAs' bytes); each CTA's
scale atoms complete on its own sf_land barrier (a low-rank slot's producer completes that phase at
once); the writers wait for sf_land only, store the scales and arrive on the even CTA's sf_full;
the issuer waits for full and sf_full, issues the MMAs and commits to both CTAs' empty barriers.
At the end each producer waits for the release of every slot it filled, so no copy is in flight
when its CTA exits.

Both accumulator modes are covered: one 256- or 192-column buffer (NVFP4, 5-stage ring, 4 scale
buffers), one 384-column buffer (NVFP4, 4-stage ring, 2 scale buffers), and two buffers used
alternately (NVFP4 128-wide tiles with a 6-stage ring, and every FP8 tile width with 6- and 8-stage
rings, where without scale factors the issuer waits on the full barrier alone).
Checked: no deadlock, no stray arrival, waits on exactly their completion, no resource used before
its previous user is done; removing any one wait must make it fail."""
import random

import pytest

WAITS = ["producer.empty", "producer.drain", "issuer.acce", "issuer.full", "issuer.sf_full", "sf.land",
         "sf.release", "epi.accf"]


class Barrier:
    def __init__(self, name, count):
        self.name, self.count, self.pending, self.completed = name, count, count, 0

    def arrive(self, n=1):
        self.pending -= n
        assert self.pending >= 0, f"{self.name}: more arrivals than its count in one phase"
        if self.pending == 0:
            self.completed += 1
            self.pending = self.count


def run_model(n_tiles, r, k_iters, stages, acc_bufs, seed, skip=(), scales=True, sf_bufs=4):
    SF_BUFS = sf_bufs
    rng = random.Random(seed)
    lr_slots = (r + 31) // 32
    slots = lr_slots + k_iters
    B = {}

    def bar(name, count):
        B[name] = Barrier(name, count)

    for s in range(stages):
        bar(f"full.{s}", 3)          # the even producer's arrive + the landing of each CTA's copies
    for c in (0, 1):
        for s in range(stages):
            bar(f"empty{c}.{s}", 1)
            bar(f"sf_land{c}.{s}", 2)  # the producer's arrive + the landing of the scale atoms
        for a in range(acc_bufs):
            bar(f"accf{c}.{a}", 1)
    for a in range(acc_bufs):
        bar(f"acce{a}", 16)
    for b in range(SF_BUFS):
        bar(f"sf_full{b}", 8)
    done = lambda name: B[name].completed  # noqa: E731
    in_flight = []
    issued = {c: [0] * stages for c in (0, 1)}
    landed = {c: [0] * stages for c in (0, 1)}

    def land(c, s):
        def f():
            landed[c][s] += 1
            B[f"full.{s}"].arrive()
        return f

    def arrive(name):
        return lambda: B[name].arrive()

    def wait(tag, name, index):
        if tag in skip:
            return
        while (B[name].completed & 1) == (index & 1):
            yield name
        assert B[name].completed == index + 1, \
            f"{name}: wait for completion #{index} passed at completed = {B[name].completed}"

    def producer(c):
        uses = [0] * stages
        stage = 0
        for g in range(n_tiles * slots):
            has_sf = g % slots >= lr_slots
            yield from wait("producer.empty", f"empty{c}.{stage}", uses[stage] - 1)
            assert done(f"empty{c}.{stage}") >= uses[stage], "ring stage refilled while its MMAs read it"
            uses[stage] += 1
            if scales:
                if has_sf:
                    B[f"sf_land{c}.{stage}"].arrive()
                    in_flight.append(arrive(f"sf_land{c}.{stage}"))
                else:
                    B[f"sf_land{c}.{stage}"].arrive(2)
            if c == 0:
                B[f"full.{stage}"].arrive()
            issued[c][stage] += 1
            in_flight.append(land(c, stage))
            stage = (stage + 1) % stages
        for s in range(stages):
            if uses[s]:
                yield from wait("producer.drain", f"empty{c}.{s}", uses[s] - 1)
        assert landed[c] == issued[c], "CTA may exit with a copy in flight"

    def issuer():
        stage, sfb, g = 0, 0, 0
        sf_uses = [0] * SF_BUFS
        for t in range(n_tiles):
            a, use = t % acc_bufs, t // acc_bufs
            yield from wait("issuer.acce", f"acce{a}", use - 1)
            assert done(f"acce{a}") >= use, "accumulator overwritten before its epilogue read it"
            for _ in range(slots):
                yield from wait("issuer.full", f"full.{stage}", g // stages)
                if scales:
                    yield from wait("issuer.sf_full", f"sf_full{sfb}", sf_uses[sfb])
                    sf_uses[sfb] += 1
                for c in (0, 1):
                    assert landed[c][stage] >= g // stages + 1, "MMA before a CTA's copy landed"
                    if scales:
                        assert stored[c][g] if g < len(stored[c]) else False, "MMA before a CTA stored its scales"
                for c in (0, 1):
                    in_flight.append(arrive(f"empty{c}.{stage}"))
                stage = (stage + 1) % stages
                sfb = (sfb + 1) % SF_BUFS
                g += 1
            for c in (0, 1):
                in_flight.append(arrive(f"accf{c}.{a}"))

    stored = {c: [] for c in (0, 1)}

    def sf_writers(c):
        land_uses = [0] * stages
        released = [0] * stages
        stage, sfb, n = 0, 0, 0
        for g in range(n_tiles * slots):
            yield from wait("sf.land", f"sf_land{c}.{stage}", land_uses[stage])
            land_uses[stage] += 1
            has_sf = g % slots >= lr_slots
            if has_sf:
                assert done(f"sf_land{c}.{stage}") >= land_uses[stage], "scales read before they landed"
            if n >= SF_BUFS:
                ps = (stage - SF_BUFS) % stages
                yield from wait("sf.release", f"empty{c}.{ps}", released[ps])
                released[ps] += 1
            # the scale buffer this slot writes was last read by the MMAs of slot n - SF_BUFS
            assert n < SF_BUFS or done(f"empty{c}.{(stage - SF_BUFS) % stages}") >= \
                (n - SF_BUFS) // stages + 1, "scale buffer rewritten while its MMAs read it"
            stored[c].append(True)
            B[f"sf_full{sfb}"].arrive(4)
            n += 1
            stage = (stage + 1) % stages
            sfb = (sfb + 1) % SF_BUFS

    def epilogue(c):
        for t in range(n_tiles):
            a, use = t % acc_bufs, t // acc_bufs
            yield from wait("epi.accf", f"accf{c}.{a}", use)
            assert done(f"accf{c}.{a}") >= use + 1, "accumulator read before its MMAs completed"
            B[f"acce{a}"].arrive()

    live = {"issuer": issuer()}
    for c in (0, 1):
        live[f"producer{c}"] = producer(c)
        if scales:
            live[f"sf{c}"] = sf_writers(c)
        for w in range(8):
            live[f"epi{c}.{w}"] = epilogue(c)

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
            in_flight.pop()()
    assert not live, "model did not finish"
    while in_flight:
        in_flight.pop()()
    for name, b in B.items():
        assert b.pending == b.count, f"{name}: {b.count - b.pending} stray arrivals at the end"
    return True


# (stages, accumulator buffers, scale factors, scale buffers) of the kernel's instantiations:
# NVFP4 256 / 192 -> (5, 1, 4 buffers), NVFP4 384 -> (4, 1, 2 buffers), NVFP4 128 -> (6, 2, 4
# buffers); row-wise FP8 256 / 192 -> (6, 2, no scales), 128 -> (8, 2, no scales)
MODES = [(5, 1, True, 4), (4, 1, True, 2), (6, 2, True, 4), (6, 2, False, 4), (8, 2, False, 4)]


@pytest.mark.parametrize("stages,acc_bufs,scales,sf_bufs", MODES)
@pytest.mark.parametrize("n_tiles", [1, 2, 3, 8])
@pytest.mark.parametrize("r,k_iters", [(32, 1), (64, 2), (0, 3), (16, 12)])
def test_pair_gemm_protocol_model(stages, acc_bufs, scales, sf_bufs, n_tiles, r, k_iters):
    for seed in range(5):
        assert run_model(n_tiles, r, k_iters, stages, acc_bufs, seed, scales=scales, sf_bufs=sf_bufs)


@pytest.mark.parametrize("skipped", WAITS)
@pytest.mark.parametrize("stages,acc_bufs,scales,sf_bufs", MODES)
def test_every_wait_is_needed(skipped, stages, acc_bufs, scales, sf_bufs):
    if not scales and skipped.startswith(("sf.", "issuer.sf_")):
        pytest.skip("no scale factors in this format")
    for n_tiles in (3, 8):
        for r, k_iters in ((32, 1), (0, 3), (16, 12)):
            for seed in range(20):
                try:
                    run_model(n_tiles, r, k_iters, stages, acc_bufs, seed, skip={skipped}, scales=scales,
                              sf_bufs=sf_bufs)
                except AssertionError:
                    return
    pytest.fail(f"removing the wait {skipped} went unnoticed")
