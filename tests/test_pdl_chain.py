"""The programmatic-dependent-launch chain of the library's calls, restated as a
small model and checked over sequences of calls.  CPU only.

Every kernel of the library waits (griddepcontrol.wait) for its predecessor on the
stream before it reads or writes anything a predecessor touches, except the reads
it does before that wait.  A kernel lets its successor launch at one of three
points: at its entry, right after its own wait, or only at its exit (no trigger).
What that guarantees:

  - a kernel's wait returns once its predecessor has completed, and a kernel
    completes after its own wait, so when kernel k completes, every earlier kernel
    has completed;
  - kernel j launches after kernel j-1 triggered: if j-1 triggers at its exit,
    kernels 0..j-1 have completed; after its wait, kernels 0..j-2; at its entry,
    whatever had completed when j-1 itself launched.

A read before the wait is safe when every earlier kernel that writes that resource
has completed by the reader's launch.  The model lists, per kernel of each call,
its trigger point, the resources it reads before its wait and the resources it
writes; the check runs over every sequence of two and three calls.  A second check
shows that the standalone append and absorb must not trigger after their wait (the
mode they had before the decodes read the cache rows and queries early).
"""
import itertools

import pytest

ENTRY, AFTER_WAIT, EXIT = "entry", "after-wait", "exit"


def calls(append_trigger=EXIT, absorb_trigger=EXIT):
    """Kernels per call: (name, trigger point, reads before the wait, writes).
    Resources: 'cache' (rows other than a fused step's own new slots), 'new:S'
    (the new slots of call S), 'q_abs', 'q_rot', 'partials', 'out'."""
    def c(tag):
        return {
            "append": [("append", append_trigger, {"in"}, {f"new:{tag}", "cache"})],
            "absorb": [("absorb", absorb_trigger, {"in"}, {"q_abs"})],
            "decode": [("split", AFTER_WAIT, {"in", "cache", "q_abs"}, {"partials"}),
                       ("combine", ENTRY, {"in"}, {"out"})],
            "step": [("prep", ENTRY, {"in"}, {f"new:{tag}", "q_abs"}),
                     ("split", AFTER_WAIT, {"in", "cache"}, {"partials"}),
                     ("combine", ENTRY, {"in"}, {"out"})],
            "gqa_append": [("gqa_append", append_trigger, {"in"}, {f"new:{tag}", "cache"})],
            "gqa_decode": [("split", AFTER_WAIT, {"in", "cache", "q_rot"}, {"partials"}),
                           ("combine", ENTRY, {"in"}, {"out"})],
            "gqa_step": [("gqa_prep", ENTRY, {"in"}, {f"new:{tag}", "q_rot"}),
                         ("split", AFTER_WAIT, {"in", "cache"}, {"partials"}),
                         ("combine", ENTRY, {"in"}, {"out"})],
        }
    return c


def kernels_of(seq, c):
    ks = []
    for i, call in enumerate(seq):
        ks += c(i)[call]
    return ks


def violations(ks):
    """(reader, resource, writer) triples where a read before the wait may see an
    incomplete write."""
    n = len(ks)
    done_at_launch = [set() for _ in range(n)]
    for j in range(1, n):
        trig = ks[j - 1][1]
        if trig == EXIT:
            done_at_launch[j] = set(range(j))
        elif trig == AFTER_WAIT:
            done_at_launch[j] = set(range(j - 1))
        else:
            done_at_launch[j] = set(done_at_launch[j - 1])
    bad = []
    for j, (name, _, reads, _) in enumerate(ks):
        for i in range(j):
            writes = ks[i][3]
            for r in reads:
                # "cache" rows read early are the rows other than a fused step's own
                # new slots; any earlier writer of cache rows counts
                if (r in writes or (r == "cache" and any(w.startswith("new:") for w in writes))) \
                        and i not in done_at_launch[j]:
                    bad.append((j, name, r, i, ks[i][0]))
    return bad


CALLS = ["append", "absorb", "decode", "step", "gqa_append", "gqa_decode", "gqa_step"]


@pytest.mark.parametrize("length", [2, 3])
def test_every_early_read_sees_complete_writes(length):
    c = calls()
    for seq in itertools.product(CALLS, repeat=length):
        ks = kernels_of(seq, c)
        # within a fused step the split reads only rows other than its prep's new
        # slots before its wait: drop that one pair, which the kernel handles itself
        bad = [v for v in violations(ks)
               if not (ks[v[3]][0] in ("prep", "gqa_prep") and v[0] == v[3] + 1)]
        assert not bad, (seq, bad)


def test_appends_and_absorb_triggering_after_their_wait_would_race():
    """With the standalone append or absorb triggering right after its wait (before
    its stores), a decode issued next reads cache rows or queries too early."""
    for kind, seq, res in (("append", ("append", "decode"), "cache"),
                           ("absorb", ("absorb", "decode"), "q_abs"),
                           ("append", ("gqa_append", "gqa_decode"), "cache")):
        c = calls(append_trigger=AFTER_WAIT) if kind == "append" else calls(absorb_trigger=AFTER_WAIT)
        bad = violations(kernels_of(seq, c))
        assert any(v[2] == res for v in bad), (seq, bad)


def test_fused_step_split_must_not_read_its_own_new_slots_early():
    """The one pair the split kernel handles itself: its prep (triggering at entry)
    may still be writing the step's new slots and queries when it starts, which is
    why it skips tiles holding those slots before its wait and reads the queries
    after it."""
    ks = kernels_of(("step",), calls())
    bad = violations(ks)
    assert any(v[1] == "split" and v[4] == "prep" for v in bad)
