"""Model of the row-gather pipeline's shared-memory ring (csrc/gather.cu).

One producer fills jobs 0, 1, 2, ... in order; job n uses stage n % S and is
consumed by warp n % W (W = 4 consumer warps); the producer may refill a
stage only after that stage's previous job was released; the bulk copies of
different jobs complete in any order.  A consumer waiting for job n tests
the stage's mbarrier with parity (n // S) & 1, which passes as soon as the
barrier's number of completed phases has the other parity.

The model checks the design rule the kernel relies on: with S a multiple of
W every stage has a single consumer and the parity test never passes before
job n's copies have landed; with S = 5 (not a multiple of 4) a schedule
exists where it passes early (a warp would read a stage whose previous job,
consumed by another warp, is still being written)."""
import random

W = 4


def run(S, n_jobs, seed):
    """Random schedule; returns True if some parity wait passed early."""
    rng = random.Random(seed)
    completed = [0] * S            # completed phases (fills) per stage
    released = set()               # jobs whose consumer released the stage
    filled = set()                 # jobs whose fill completed
    in_flight = []                 # issued fills not yet completed
    next_fill = 0
    next_job = list(range(W))      # each warp's next job
    early = False
    while any(j < n_jobs for j in next_job):
        actions = []
        prev = next_fill - S
        if next_fill < n_jobs and (prev < 0 or prev in released):
            actions.append("issue")
        if in_flight:
            actions.append("complete")
        for w in range(W):
            n = next_job[w]
            if n < n_jobs and (completed[n % S] & 1) != ((n // S) & 1):
                actions.append(("consume", w))
        assert actions, "deadlock"
        a = rng.choice(actions)
        if a == "issue":
            in_flight.append(next_fill)
            next_fill += 1
        elif a == "complete":
            n = in_flight.pop(rng.randrange(len(in_flight)))
            completed[n % S] += 1
            filled.add(n)
        else:
            w = a[1]
            n = next_job[w]
            if n not in filled:
                early = True       # the parity test passed on an older phase
                filled.add(n)      # (model: the warp goes on with stale data)
            released.add(n)
            next_job[w] += W
    return early


def test_stage_count_multiple_of_consumer_warps_never_passes_early():
    for S in (4, 8):
        for seed in range(300):
            assert not run(S, 64, seed), (S, seed)


def test_five_stages_can_pass_early():
    assert any(run(5, 64, seed) for seed in range(300))
