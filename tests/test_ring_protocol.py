"""Model of the row-gather pipeline's shared-memory ring (csrc/gather.cu).

P producer warps fill the jobs: job n uses stage n % S, is armed by producer
n % P (each producer arms its own jobs in order) and is consumed by warp
n % W (W = 4 consumer warps); the bulk copies of different jobs complete in
any order.  Both sides wait on a stage's mbarrier by parity, which passes as
soon as the barrier's number of completed phases has the awaited parity:
  * a consumer of job n waits on the stage's fill barrier with parity
    (n // S) & 1, passing once the fills completed on the stage reach the
    other parity;
  * the producer of job n waits on the stage's release barrier with parity
    ((n // S) & 1) ^ 1, passing once the releases of the stage have the
    parity of n // S.

The model checks the design rule the kernel relies on: with S a multiple of
W and of P every stage has a single producer and a single consumer, and no
parity test passes before the event it waits for (job n's copies landed, or
job n - S released).  With S = 5 (not a multiple of 4) a stage has several
consumers and schedules go wrong: a wait passes early (a warp would read a
stage whose previous job, consumed by another warp, is still being written)
or every side stalls; with two producers and S odd or not a multiple of 4,
the same."""
import random

W = 4


def run(S, n_jobs, seed, P=1):
    """Random schedule; returns "early" if some parity wait passed early,
    "stuck" if no side can move before every job is consumed, else "ok"."""
    rng = random.Random(seed)
    completed = [0] * S            # completed phases (fills) per stage
    releases = [0] * S             # completed phases (releases) per stage
    released = set()               # jobs whose consumer released the stage
    filled = set()                 # jobs whose fill completed
    in_flight = []                 # issued fills not yet completed
    next_fill = list(range(P))     # each producer's next job
    next_job = list(range(W))      # each warp's next job
    early = False
    while any(j < n_jobs for j in next_job):
        actions = []
        for p in range(P):
            n = next_fill[p]
            if n < n_jobs and (releases[n % S] & 1) == ((n // S) & 1):
                actions.append(("issue", p))
        if in_flight:
            actions.append(("complete",))
        for w in range(W):
            n = next_job[w]
            if n < n_jobs and (completed[n % S] & 1) != ((n // S) & 1):
                actions.append(("consume", w))
        if not actions:
            return "stuck"
        a = rng.choice(actions)
        if a[0] == "issue":
            n = next_fill[a[1]]
            if n >= S and n - S not in released:
                early = True       # the stage is refilled while still in use
            in_flight.append(n)
            next_fill[a[1]] += P
        elif a[0] == "complete":
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
            releases[n % S] += 1
            next_job[w] += W
    return "early" if early else "ok"


def test_stage_count_multiple_of_consumer_warps_never_passes_early():
    for S in (4, 8):
        for seed in range(300):
            assert run(S, 64, seed) == "ok", (S, seed)


def test_several_producers_never_pass_early():
    """Two or four producer warps (job n armed by warp n % P); the kernel uses four."""
    for P in (2, 4):
        for S in (4, 8):
            for seed in range(300):
                assert run(S, 64, seed, P=P) == "ok", (P, S, seed)


def test_five_stages_go_wrong():
    assert any(run(5, 64, seed) != "ok" for seed in range(300))


def test_two_producers_need_a_stage_count_multiple_of_four():
    """S odd (a stage with two producers) or S = 6 (two consumers): schedules
    pass early; likewise four producers on 6 stages."""
    for S, P in ((9, 2), (6, 2), (6, 4)):
        assert any(run(S, 64, seed, P=P) == "early" for seed in range(300)), (S, P)
