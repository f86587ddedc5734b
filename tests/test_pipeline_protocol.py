"""A model of the barrier protocol of the decode GEMM kernel
(fp4_block_scaled_route_b200/csrc/moe_gemm.cu), and at the end of the file
of the MXFP8 token-major kernel (moe_gemm_tmx.cu), run under random
interleavings on the CPU.

Agents, as in the kernel:
  - NPROD producer warps; warp p takes the pipeline iterations it with
    it % NPROD == p.  For it >= STAGES it waits for the MMAs of
    it - STAGES (mdone ring, NMD = STAGES + NBUF barriers), then posts the
    stage's transaction count on full[it % STAGES]; the bytes land later.
  - NMMA MMA warps; warp m takes it % NMMA == m, waits for its accumulator
    (tempty[it % NBUF], released by the epilogue) and for its stage
    (full[it % STAGES]), issues, and its commit later arrives on
    mdone[it % NMD].
  - The epilogue takes every iteration in order: waits on mdone, then
    releases the accumulator.

Barriers follow mbarrier parity semantics: a wait for parity P passes when
the number of completed phases has parity != P.  The model records a
violation when an MMA warp passes its stage wait before that iteration's
bytes landed, when a producer posts on a phase that already has a post, or
when the epilogue passes before the iteration's MMAs completed.

The kernel's stage-ring rule is: STAGES a multiple of NMMA, or
NBUF <= STAGES (and STAGES >= NPROD).  The model finds a violation quickly
for the configuration that breaks it (3 stages, 4 accumulators, two MMA
warps) and none for the configurations the kernel builds.
"""
import random

import pytest


class Barrier:
    """mbarrier with one expected arrival per phase (and, for a stage
    barrier, the bytes of one iteration)."""

    def __init__(self):
        self.completed = 0
        self.posted = False   # arrive.expect_tx of the current phase happened
        self.pending = 0      # iterations whose bytes the current phase waits for

    def passes(self, parity):
        return (self.completed & 1) != parity

    def arrive(self):
        self.completed += 1


def run(STAGES, NBUF, NPROD=3, NMMA=2, iters=48, seed=0):
    """One random schedule; returns the list of violations."""
    rng = random.Random(seed)
    NMD = STAGES + NBUF
    full = [Barrier() for _ in range(STAGES)]
    mdone = [Barrier() for _ in range(NMD)]
    tempty = [Barrier() for _ in range(NBUF)]
    landed = set()
    mma_done = set()
    violations = []

    prod_next = list(range(NPROD))            # next iteration per producer warp
    mma_next = list(range(NMMA))              # next iteration per MMA warp
    epi_next = [0]
    in_flight_bytes = []                      # iterations posted whose bytes have not landed
    in_flight_mma = []                        # iterations issued whose commit has not arrived

    def full_land(it):
        b = full[it % STAGES]
        landed.add(it)
        b.pending -= 1
        if b.posted and b.pending == 0:
            b.posted = False
            b.arrive()

    def step():
        actions = []
        for p in range(NPROD):
            it = prod_next[p]
            if it >= iters:
                continue
            if it >= STAGES:
                prev = it - STAGES
                if not mdone[prev % NMD].passes((prev // NMD) & 1):
                    continue
            actions.append(("prod", p))
        for m in range(NMMA):
            it = mma_next[m]
            if it >= iters:
                continue
            if not tempty[it % NBUF].passes(((it // NBUF) & 1) ^ 1):
                continue
            if not full[it % STAGES].passes((it // STAGES) & 1):
                continue
            actions.append(("mma", m))
        it = epi_next[0]
        if it < iters and mdone[it % NMD].passes((it // NMD) & 1):
            actions.append(("epi", 0))
        for i in range(len(in_flight_bytes)):
            actions.append(("land", i))
        for i in range(len(in_flight_mma)):
            actions.append(("commit", i))
        if not actions:
            return False
        kind, idx = rng.choice(actions)
        if kind == "prod":
            it = prod_next[idx]
            b = full[it % STAGES]
            if b.posted:
                violations.append(("second post on an incomplete phase", it))
            b.posted = True
            b.pending += 1
            in_flight_bytes.append(it)
            prod_next[idx] += NPROD
        elif kind == "mma":
            it = mma_next[idx]
            if it not in landed:
                violations.append(("MMA passed its stage before the bytes landed", it))
            in_flight_mma.append(it)
            mma_next[idx] += NMMA
        elif kind == "epi":
            it = epi_next[0]
            if it not in mma_done:
                violations.append(("epilogue passed before the MMAs completed", it))
            tempty[it % NBUF].arrive()
            epi_next[0] += 1
        elif kind == "land":
            # bytes land in any order
            full_land(in_flight_bytes.pop(idx))
        else:
            # commits of one MMA warp complete in its issue order
            it = in_flight_mma[idx]
            warp = it % NMMA
            first = min(j for j in in_flight_mma if j % NMMA == warp)
            in_flight_mma.remove(first)
            mma_done.add(first)
            mdone[first % NMD].arrive()
        return True

    for _ in range(100000):
        if not step() or violations:
            break
    return violations


def rule_holds(STAGES, NBUF, NPROD=3, NMMA=2):
    return (STAGES % NMMA == 0 or NBUF <= STAGES) and STAGES >= NPROD


# (STAGES, NBUF) of the kernel's instantiations: FP8 and MXFP4 decode (6, 8),
# 32-token tiles (5, 4), GEMM2 single tiles (11 or 12, 8), NVFP4 four tiles
# (5, 4), MXFP4 four-tile GEMM2 with the accumulator cap (3, 3)
BUILT = [(6, 8), (5, 4), (11, 8), (12, 8), (10, 8), (5, 2), (3, 3), (6, 4), (20, 8)]


@pytest.mark.parametrize("STAGES,NBUF", BUILT)
def test_built_configurations_keep_the_protocol(STAGES, NBUF):
    assert rule_holds(STAGES, NBUF)
    for seed in range(150):
        assert run(STAGES, NBUF, seed=seed) == [], (STAGES, NBUF, seed)


@pytest.mark.parametrize("STAGES,NBUF", [(3, 4), (5, 8), (3, 8)])
def test_odd_stage_ring_below_the_accumulators_breaks(STAGES, NBUF):
    """The rule's first clause is necessary: with an odd stage count below
    NBUF an MMA warp can pass a stage on its phase before last."""
    assert not rule_holds(STAGES, NBUF)
    found = [v for seed in range(400) for v in run(STAGES, NBUF, seed=seed)]
    assert any(v[0].startswith("MMA passed") for v in found), found[:3]


def test_token_major_kernel_keeps_the_protocol():
    """moe_gemm_tm.cu: 4 stages, 2 accumulators, 2 producer warps."""
    assert rule_holds(4, 2, NPROD=2)
    for seed in range(150):
        assert run(4, 2, NPROD=2, seed=seed) == []


def test_one_mma_warp_needs_no_rule():
    """With a single MMA warp every iteration sharing a stage is its own."""
    for seed in range(150):
        assert run(3, 8, NMMA=1, seed=seed) == []


@pytest.mark.parametrize("STAGES,NBUF,NPROD", [(2, 2, 3), (4, 2, 5)])
def test_fewer_stages_than_producers_breaks(STAGES, NBUF, NPROD):
    """The second clause: with fewer stages than producer warps a producer's
    wait on the MMA-done ring can pass on a stale phase and post twice."""
    assert not rule_holds(STAGES, NBUF, NPROD=NPROD)
    found = [v for seed in range(400) for v in run(STAGES, NBUF, NPROD=NPROD, seed=seed)]
    assert any(v[0].startswith("second post") for v in found), found[:3]


# ---- the MXFP8 token-major kernel (moe_gemm_tmx.cu) -------------------------------
def run_tmx(STAGES, KB, units=5, NPROD=2, unit_barrier=True, seed=0):
    """One random schedule of the MXFP8 kernel's protocol.  Producers as
    above; one MMA warp takes every iteration in order and, at a unit's first
    K block, waits for the epilogue to have read the one accumulator (tempty,
    one phase per unit); each iteration's commit arrives on mdone[it % NMD]
    (NMD = STAGES + 1), and the unit's last one also on the unit barrier
    afull.  The epilogue waits once per unit, on afull (unit_barrier) or, as
    a first version of the kernel did, on the ring barrier of the unit's last
    iteration; then it releases the accumulator."""
    rng = random.Random(seed)
    NMD = STAGES + 1
    iters = units * KB
    full = [Barrier() for _ in range(STAGES)]
    mdone = [Barrier() for _ in range(NMD)]
    afull, tempty = Barrier(), Barrier()
    landed, mma_done, violations = set(), set(), []
    prod_next = list(range(NPROD))
    mma_next, epi_unit = [0], [0]
    in_flight_bytes, in_flight_mma = [], []

    def epi_passes(j):
        last = j * KB + KB - 1
        if unit_barrier:
            return afull.passes(j & 1)
        return mdone[last % NMD].passes((last // NMD) & 1)

    def step():
        actions = []
        for p in range(NPROD):
            it = prod_next[p]
            if it < iters and (it < STAGES or mdone[(it - STAGES) % NMD].passes(((it - STAGES) // NMD) & 1)):
                actions.append(("prod", p))
        it = mma_next[0]
        if it < iters:
            j, kb = divmod(it, KB)
            if (kb != 0 or tempty.passes((j & 1) ^ 1)) and full[it % STAGES].passes((it // STAGES) & 1):
                actions.append(("mma", 0))
        if epi_unit[0] < units and epi_passes(epi_unit[0]):
            actions.append(("epi", 0))
        actions += [("land", i) for i in range(len(in_flight_bytes))]
        if in_flight_mma:
            actions.append(("commit", 0))
        if not actions:
            return False
        kind, idx = rng.choice(actions)
        if kind == "prod":
            it = prod_next[idx]
            b = full[it % STAGES]
            if b.posted:
                violations.append(("second post on an incomplete phase", it))
            b.posted, b.pending = True, b.pending + 1
            in_flight_bytes.append(it)
            prod_next[idx] += NPROD
        elif kind == "mma":
            it = mma_next[0]
            if it not in landed:
                violations.append(("MMA passed its stage before the bytes landed", it))
            in_flight_mma.append(it)
            mma_next[0] += 1
        elif kind == "epi":
            j = epi_unit[0]
            if j * KB + KB - 1 not in mma_done:
                violations.append(("epilogue read the accumulator before the unit's MMAs completed", j))
            tempty.arrive()
            epi_unit[0] += 1
        elif kind == "land":
            it = in_flight_bytes.pop(idx)
            b = full[it % STAGES]
            landed.add(it)
            b.pending -= 1
            if b.posted and b.pending == 0:
                b.posted = False
                b.arrive()
        else:
            it = in_flight_mma.pop(0)  # one warp: commits complete in issue order
            mma_done.add(it)
            mdone[it % NMD].arrive()
            if it % KB == KB - 1:
                afull.arrive()
        return True

    for _ in range(200000):
        if not step() or violations:
            break
    return violations


@pytest.mark.parametrize("KB", [1, 2, 4, 5, 6, 8, 16])
def test_mxfp8_kernel_keeps_the_protocol(KB):
    """moe_gemm_tmx.cu as built: 4 stages, 2 producer warps, the unit barrier."""
    for seed in range(100):
        assert run_tmx(4, KB, seed=seed) == [], (KB, seed)


def test_mxfp8_epilogue_on_the_ring_barrier_breaks_past_the_ring():
    """With more K blocks per unit than ring slots, a parity wait on the ring
    barrier of the unit's last iteration can pass on an earlier phase: the
    failure the MXFP8 kernel first had (H >= 768 at 4 stages)."""
    assert all(run_tmx(4, 5, unit_barrier=False, seed=s) == [] for s in range(100))  # within the ring: exact
    found = [v for seed in range(200) for v in run_tmx(4, 6, unit_barrier=False, seed=seed)]
    assert any(v[0].startswith("epilogue read") for v in found), found[:3]
