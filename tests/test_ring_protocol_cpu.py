"""The activation kernel's stage ring as a model on the CPU: one producer, G groups of
converter warps that take alternate chunks (group g converts chunks i with i % G == g), and
the MMA thread, over S stages guarded by mbarriers waited on by phase parity.

An mbarrier here is a phase counter phi: a wait for parity p passes when (phi & 1) != p, i.e.
when the phase of that parity has completed (so a fresh barrier passes a wait for parity 1).
Loads land, and MMA commits arrive, in any order after they are issued, as the copy engine and
the tensor pipe allow.  A random scheduler explores the interleavings; every consumer checks
that the stage it reads holds the chunk it expects.

The kernel's layouts (S = 4, G = 1; S = 8 or 6, G = 2) never read a stale stage and always
finish.  A stage count that is not a multiple of G lets a group pass a parity wait one phase
early (its stage is shared with the other group, whose load has not landed yet): the model
finds that, which is why the kernel asserts S % G == 0."""

import random

import pytest


def run_ring(S, G, nchunks, seed, max_steps=200000):
    """Returns (finished, violations)."""
    rng = random.Random(seed)
    phi = {("FULL", s): 0 for s in range(S)}
    phi.update({("CONV", s): 0 for s in range(S)})
    phi.update({("EMPTY", s): 0 for s in range(S)})
    content = [None] * S            # chunk whose data sits in stage s
    pending = []                    # ("load", s, chunk) or ("commit", s)
    violations = []

    def passes(bar, parity):
        return (phi[bar] & 1) != parity

    # program counters
    prod_i = 0
    group_next = [g for g in range(G)]   # next chunk of each group
    mma_i = 0
    mma_got_conv = False

    for _ in range(max_steps):
        actions = []
        if prod_i < nchunks:
            s, ph = prod_i % S, (prod_i // S) & 1
            if passes(("EMPTY", s), ph ^ 1):
                actions.append("prod")
        for g in range(G):
            i = group_next[g]
            if i < nchunks and passes(("FULL", i % S), (i // S) & 1):
                actions.append(("conv", g))
        if mma_i < nchunks:
            s, ph = mma_i % S, (mma_i // S) & 1
            if not mma_got_conv and passes(("CONV", s), ph):
                actions.append("mma_conv")
            elif mma_got_conv and passes(("FULL", s), ph):
                actions.append("mma")
        actions.extend(("land", k) for k in range(len(pending)))
        if not actions:
            done = prod_i == nchunks and mma_i == nchunks and all(i >= nchunks for i in group_next) and not pending
            return done, violations
        a = rng.choice(actions)
        if a == "prod":
            s = prod_i % S
            pending.append(("load", s, prod_i))
            prod_i += 1
        elif a == "mma_conv":
            mma_got_conv = True
        elif a == "mma":
            s = mma_i % S
            if content[s] != mma_i:
                violations.append(("mma reads", mma_i, content[s]))
            pending.append(("commit", s))
            mma_i += 1
            mma_got_conv = False
        elif a[0] == "conv":
            g = a[1]
            i = group_next[g]
            s = i % S
            if content[s] != i:
                violations.append(("group", g, "reads", i, "stage holds", content[s]))
            phi[("CONV", s)] += 1  # the group's 256 arrivals, as one
            group_next[g] = i + G
        else:
            ev = pending.pop(a[1])
            if ev[0] == "load":
                _, s, chunk = ev
                content[s] = chunk
                phi[("FULL", s)] += 1
            else:
                phi[("EMPTY", ev[1])] += 1
    raise AssertionError("the model did not settle")


@pytest.mark.parametrize("S,G", [(4, 1), (8, 2), (6, 2), (4, 2)])
def test_kernel_layouts_never_read_a_stale_stage(S, G):
    """(4, 1), (8, 2), (6, 2): the activation kernel's instances.  (4, 2): the INT4 GEMM's ring,
    whose two widening groups take alternate stages the same way (they wait for the landed codes,
    widen them and arrive on the stage's barrier for the MMA thread)."""
    for nchunks in list(range(1, 20)) + [24, 48, 64]:
        for seed in range(40):
            done, bad = run_ring(S, G, nchunks, seed=1000 * nchunks + seed)
            assert done, (S, G, nchunks, seed, "deadlock")
            assert not bad, (S, G, nchunks, seed, bad[:3])


@pytest.mark.parametrize("S,G", [(5, 2), (6, 4)])
def test_a_stage_count_not_a_multiple_of_the_groups_reads_stale_data(S, G):
    """The planted fault: stages shared by two groups let a parity wait alias."""
    found = False
    for nchunks in (16, 24, 40):
        for seed in range(400):
            done, bad = run_ring(S, G, nchunks, seed=seed)
            if bad:
                found = True
                break
        if found:
            break
    assert found
