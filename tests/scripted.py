"""Scripted row models for pinning the speculative state machine.

A scripted model has no numerics: its readout at depth r for a prefix returns
logits whose argmax a script chooses, so the schedule's loop-step counts can be
compared with the worked example of the LoopSpec page (section 2.2, Fig. 1)
and with the branch count of section 3.4.
"""
import numpy as np


class ScriptedRows:
    def __init__(self, vocab, script):
        self.V = vocab
        self.script = script  # script(prefix tuple, depth) -> token id

    def prelude(self, prefix, pos, slots):
        return None

    def iterate(self, h, r, prefix, pos, slots):
        return None

    def readout(self, h, r, prefix, pos, slots, head=True):
        if not head:
            return None
        z = np.zeros(self.V)
        z[self.script(tuple(int(t) for t in prefix), r)] = 1.0
        return z


# Fig. 1 vocabulary.  The prompt is [8, 9]; prefill commits "is", after which
# the three tokens of the figure are decoded: "Paris", "and", "it".
IS, FRANCE, PARIS, AND, IT, THE, OTHER = 1, 2, 3, 4, 5, 6, 7
FIG1_PROMPT = [8, 9]


def fig1_script(first_it: bool):
    """Depth-1 readout after "is" says "France", deeper ones "Paris".
    first_it: the depth-1 readout after "Paris and" already says "it" (all
    accepted, as in the left panel); otherwise it says "the" and only deeper
    readouts say "it" (the right panel's pruned "the" subtree)."""
    def s(prefix, r):
        if len(prefix) <= len(FIG1_PROMPT):
            return IS
        tail = prefix[len(FIG1_PROMPT) + 1:]
        if tail == ():
            return FRANCE if r == 1 else PARIS
        if tail == (PARIS,):
            return AND
        if tail == (PARIS, AND):
            return IT if (first_it or r >= 2) else THE
        return OTHER
    return s


def fork_script(d2: int):
    """Every readout proposes token 1 and full depth confirms it, except the
    depth-d2 readout, which prefers token 2: with greedy readouts the gate opens
    at every d2 and the first proposal is always accepted (unconditional
    forking at both depths)."""
    def s(prefix, r):
        return 2 if r == d2 else 1
    return s
