"""A model check of the expert-parallel step protocol (the order of the moe_ep_* kernels
and the flags each waits for), on CPU.

P ranks run S steps of notify -> layout -> dispatch -> expert FFN -> combine, each stage
modelled as one atomic event with the same waits and the same remote writes as the
kernels:
  notify   writes row r of every rank's count table, then raises cnt_flag[r] everywhere
  layout   waits until every rank's cnt_flag >= s, reads its own count table
  dispatch writes its rows into the owners' receive buffers, raises disp_flag[r] everywhere
  ffn      waits until every disp_flag >= s, reads its receive buffer, writes its output
           rows, raises done_flag[r] everywhere
  combine  waits until every done_flag >= s, reads every owner's output rows
Random schedules pick any rank whose next stage may run.  The checks: nothing a rank
reads was overwritten by a later step first (one window serves every step), and no
schedule deadlocks.  Weakened protocols (a combine that does not wait, a layout that
waits only for the ranks sending to it, an owner that raises "done" before writing its
output rows) must be caught; a combine that waits only for the owners it reads from is
shown to be safe as well.  Failure propagation (a missing dispatch, a layout wait that gives
up) is checked the same way: the faulty step fails on every rank and no other step does.
"""
import numpy as np
import pytest

STAGES = ["notify", "layout", "dispatch", "ffn", "combine"]


class Violation(AssertionError):
    pass


def run_schedule(P, S, rng, sends_to, combine_waits="all", layout_waits_all=True, done_before_write=False):
    """sends_to[s][r]: the owners rank r sends rows to in step s (the count rows go to
    every rank regardless).  The keyword arguments weaken the protocol for the mutation
    tests: combine_waits "all" (the kernels), "own" (only the owners it reads from) or
    "none"; layout_waits_all False waits only for the ranks that send to this owner;
    done_before_write raises the done flags before the output rows are written."""
    cnt_flag = np.zeros((P, P), int)    # [window j][signalling rank i]
    disp_flag = np.zeros((P, P), int)
    done_flag = np.zeros((P, P), int)
    cnt_stamp = np.zeros((P, P), int)   # step that last wrote row i of window j's count table
    recv_stamp = np.zeros((P, P), int)  # step that last wrote source i's rows in window j
    out_stamp = np.zeros(P, int)        # step that last wrote window j's output rows
    read_cnt = np.zeros(P, int)         # last step whose count table rank j has read
    read_recv = np.zeros(P, int)        # last step whose receive rows rank j has read
    read_out = np.zeros((P, P), int)    # [reader i][owner j]: last step whose output rows i read
    pos = [(1, 0)] * P                  # (step, stage index) of each rank's next stage
    stages = STAGES if not done_before_write else ["notify", "layout", "dispatch", "ffn", "ffn_write", "combine"]

    def enabled(r):
        s, st = pos[r]
        if s > S:
            return False
        name = stages[st]
        if name == "layout":
            ranks = range(P) if layout_waits_all else [i for i in range(P) if r in sends_to[s][i]]
            return all(cnt_flag[r][i] >= s for i in ranks)
        if name == "ffn":
            return (disp_flag[r] >= s).all()
        if name == "ffn_write":
            return True
        if name == "combine":
            owners = {"all": range(P), "own": sends_to[s][r], "none": []}[combine_waits]
            return all(done_flag[r][j] >= s for j in owners)
        return True

    def write_out(r, s):
        for i in range(P):
            if s > 1 and read_out[i][r] < s - 1 and r in sends_to[s - 1][i]:
                raise Violation(f"step {s}: owner {r} overwrote output rows source {i} still reads")
        out_stamp[r] = s

    def step(r):
        s, st = pos[r]
        name = stages[st]
        if name == "notify":
            for j in range(P):
                if s > 1 and read_cnt[j] < s - 1:
                    raise Violation(f"step {s}: rank {r} overwrote count row in window {j} before it was read")
                cnt_stamp[j][r] = s
                cnt_flag[j][r] = s
        elif name == "layout":
            if (cnt_stamp[r] != s).any():
                raise Violation(f"step {s}: rank {r} read a count table of another step")
            read_cnt[r] = s
        elif name == "dispatch":
            for j in sends_to[s][r]:
                if s > 1 and read_recv[j] < s - 1:
                    raise Violation(f"step {s}: rank {r} overwrote receive rows of window {j} still in use")
                recv_stamp[j][r] = s
            for j in range(P):
                disp_flag[j][r] = s
        elif name == "ffn":
            for i in range(P):
                if r in sends_to[s][i] and recv_stamp[r][i] != s:
                    raise Violation(f"step {s}: owner {r} read rows of source {i} from another step")
            read_recv[r] = s
            if not done_before_write:
                write_out(r, s)
            for j in range(P):
                done_flag[j][r] = s
        elif name == "ffn_write":
            write_out(r, s)
        elif name == "combine":
            for j in sends_to[s][r]:
                if out_stamp[j] != s:
                    raise Violation(f"step {s}: rank {r} read owner {j}'s output rows of another step")
                read_out[r][j] = s
        pos[r] = (s + (st == len(stages) - 1), (st + 1) % len(stages))

    while any(p[0] <= S for p in pos):
        ready = [r for r in range(P) if enabled(r)]
        if not ready:
            raise Violation("deadlock: no rank can run its next stage")
        step(int(rng.choice(ready)))


def random_sends(P, S, rng, sparse):
    out = {}
    for s in range(1, S + 1):
        out[s] = {}
        for r in range(P):
            if sparse:
                k = int(rng.integers(1, P + 1))
                out[s][r] = set(int(j) for j in rng.choice(P, size=k, replace=False))
            else:
                out[s][r] = set(range(P))
    return out


@pytest.mark.parametrize("P", [2, 3, 4])
def test_protocol_is_safe_under_random_schedules(P):
    rng = np.random.default_rng(P)
    for trial in range(400):
        S = 3
        run_schedule(P, S, rng, random_sends(P, S, rng, sparse=trial % 2 == 1))


def test_combine_waiting_only_for_its_own_owners_is_also_safe():
    """The kernels' combine waits for every owner; waiting only for the owners it reads from
    would be enough, because the next step's layout waits for every rank's count row, and
    each rank publishes it only after finishing its combine of the step before."""
    rng = np.random.default_rng(5)
    for _ in range(400):
        run_schedule(3, 3, rng, random_sends(3, 3, rng, sparse=True), combine_waits="own")


def _caught(**weakening):
    rng = np.random.default_rng(11)
    caught = 0
    for _ in range(400):
        try:
            run_schedule(3, 3, rng, random_sends(3, 3, rng, sparse=True), **weakening)
        except Violation:
            caught += 1
    return caught


@pytest.mark.parametrize("weakening", [dict(combine_waits="none"), dict(layout_waits_all=False),
                                       dict(done_before_write=True)],
                         ids=["combine-does-not-wait", "layout-waits-for-senders-only", "done-before-write"])
def test_weakened_protocols_are_caught(weakening):
    assert _caught(**weakening) > 0


# ---------------------------------------------------------------------------------------
# Failure propagation.  Two faults: a rank that never dispatches in one step (its host
# stops before the launch), and a rank whose layout wait gives up early (a slow peer), so
# that it sends no rows that step.  Waits that can never be satisfied run out (modelled:
# when no stage of any rank can run, one of the waits that started first gives up).  A
# rank whose wait gave up fails the step, and the flags it publishes later in that step
# carry the error mark, which fails the step on every rank that waits for them.
# ---------------------------------------------------------------------------------------
def run_failing_schedule(P, S, rng, sends_to, fault, marks=True):
    """fault = (kind, step, rank), kind "skip_dispatch" or "layout_timeout".  Returns
    {(rank, step): error} of every combine.  marks=False publishes plain flags after a
    failure (the weakened protocol, in which a combine may sum rows of an owner whose
    inputs were incomplete)."""
    kind, f_step, f_rank = fault
    cnt_flag = np.zeros((P, P), int)
    disp_flag = np.zeros((P, P), int)
    done_flag = np.zeros((P, P), int)
    disp_mark = np.zeros((P, P), int)   # step whose dispatch flag carries the error mark
    done_mark = np.zeros((P, P), int)
    failed = np.zeros(P, int)           # last step that failed on each rank
    sent = {}                           # (source, step): its rows reached the owners
    owner_failed = {}                   # (owner, step): its FFN ran on incomplete inputs
    errors = {}
    pos = [(1, 0)] * P

    def enabled(r):
        s, st = pos[r]
        if s > S:
            return False
        name = STAGES[st]
        if name == "layout":
            return (cnt_flag[r] >= s).all()
        if name == "ffn":
            return (disp_flag[r] >= s).all()
        if name == "combine":
            return (done_flag[r] >= s).all()
        return True

    def step(r, timed_out=False):
        s, st = pos[r]
        name = STAGES[st]
        if name == "notify":
            for j in range(P):
                cnt_flag[j][r] = s
        elif name == "layout":
            if timed_out or (kind == "layout_timeout" and (s, r) == (f_step, f_rank)):
                failed[r] = s            # no destinations: this rank sends no rows
        elif name == "dispatch":
            if not (kind == "skip_dispatch" and (s, r) == (f_step, f_rank)):
                sent[(r, s)] = failed[r] != s
                for j in range(P):
                    disp_flag[j][r] = s
                    if marks and failed[r] == s:
                        disp_mark[j][r] = s
        elif name == "ffn":
            if timed_out or (disp_mark[r] == s).any():
                failed[r] = s
            if any(r in sends_to[s][i] and not sent.get((i, s)) for i in range(P)):
                owner_failed[(r, s)] = True
            for j in range(P):
                done_flag[j][r] = s
                if marks and failed[r] == s:
                    done_mark[j][r] = s
        elif name == "combine":
            err = timed_out or (done_mark[r] == s).any() or failed[r] == s
            if not err:
                for j in sends_to[s][r]:
                    if owner_failed.get((j, s)):
                        raise Violation(f"step {s}: rank {r} summed rows of owner {j}, whose inputs were incomplete")
            errors[(r, s)] = bool(err)
            if err:
                failed[r] = s
        pos[r] = (s + (st == len(STAGES) - 1), (st + 1) % len(STAGES))

    while any(p[0] <= S for p in pos):
        ready = [r for r in range(P) if enabled(r)]
        if ready:
            step(int(rng.choice(ready)))
            continue
        blocked = [r for r in range(P) if pos[r][0] <= S and STAGES[pos[r][1]] in ("layout", "ffn", "combine")]
        if not blocked:
            raise Violation("deadlock")
        # a bounded wait runs out: one of the oldest (earliest step and stage), which
        # started waiting first
        oldest = min(pos[r] for r in blocked)
        step(int(rng.choice([r for r in blocked if pos[r] == oldest])), timed_out=True)
    return errors


@pytest.mark.parametrize("kind", ["skip_dispatch", "layout_timeout"])
@pytest.mark.parametrize("P", [2, 3, 4])
def test_a_failed_rank_fails_that_step_on_every_rank(P, kind):
    """Every rank's combine of the faulty step reports the error (none sums an owner's
    rows computed from incomplete inputs), no other step reports one, nothing deadlocks."""
    rng = np.random.default_rng(100 + P)
    for trial in range(300):
        S = 3
        fault = (kind, int(rng.integers(1, S + 1)), int(rng.integers(0, P)))
        errors = run_failing_schedule(P, S, rng, random_sends(P, S, rng, sparse=False), fault)
        assert len(errors) == P * S
        for (r, s), err in errors.items():
            assert err == (s == fault[1]), (trial, fault, r, s)


def test_failure_without_error_marks_is_caught():
    """Without the marks, a rank whose layout gave up sends nothing, the owners do not
    notice, and the other sources sum rows computed without its tokens."""
    rng = np.random.default_rng(7)
    caught = 0
    for _ in range(300):
        fault = ("layout_timeout", int(rng.integers(1, 4)), int(rng.integers(0, 3)))
        try:
            run_failing_schedule(3, 3, rng, random_sends(3, 3, rng, sparse=False), fault, marks=False)
        except Violation:
            caught += 1
    assert caught > 0
