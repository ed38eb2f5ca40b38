"""Prefill, full-depth autoregressive decoding and the pipelined speculative
state machine -- the oracle's normative step order (test infrastructure only).

Follows "LoopSpec: Pipelined Self-Speculative Decoding for Looped Transformers"
(liuzhao09.github.io/papers/loopspec.html):
  * section 1 / 3.1: the baseline is full-depth autoregressive decoding -- each
    position runs all R loops, then commits;
  * section 2.2: after prefill the first token is committed at full depth; a
    branch is a fixed prefix plus its current loop depth; all active branches
    advance the shared block together; at depth d1 a branch reads q1 = p_d1,
    draws x1 and at once opens a child for prefix + x1; the parent continues to
    R and verifies; on acceptance the child is kept, on rejection every
    descendant of the wrong prefix is pruned and decoding restarts from the
    correct prefix; Fig. 1 gives the loop-step counts 12 / 9 / 7;
  * section 2.3: at d2 the gate of Eq. 6 decides whether a second child is
    opened with x2 ~ q2 = p_d2 (-) q1; the cascade verifies x1, then x2 against
    rho1; the tree is re-rooted on every verification; tokens with equal text
    but different prefixes are different branches;
  * section 2.4: a new branch copies its parent's cache indices (not KV);
    pruning frees only what no surviving path needs.

Step order (a reading of the pages, fixed here and followed by the CUDA
engine bit for bit):
  1. prelude for every branch at depth 0 (ascending uid);
  2. every branch runs loop iteration depth+1 (ascending uid);
  3. readouts for branches whose depth is in {d1, d2, R};
  4. proposals, ascending uid: depth == d1 -> x1 ~ q1 = p_d1, child1 (lowest
     free slot, next uid); depth == d2 and x1 drawn -> gate; if open
     x2 ~ q2 = p_d2 (-) q1, child2.  Proposals are always drawn; a child is
     created only if its own next token is still needed (pos + 1 < P + N).
     A child's first iteration is in the next step;
  5. if the root (prefix == committed) reached R: verify (cascade) and commit;
  6. prune every branch whose prefix does not extend the new committed
     sequence (its slots are freed after this step's allocations); the kept
     child becomes the root and its slot is appended to the committed slots;
     with no kept child a new root (depth 0) is created after the frees
     (unless that commit was the last one).

Context-copy proposals (CopyLoop card, kongchang.com; oracle/copy.py has the
lookup and the readings), when enabled, change steps 4-6 as follows:
  4a. a branch at depth d1 whose first proposal is a copied token (it has a
      copy child) is screened: if the token's depth-d1 score is below tau the
      copy child's subtree is pruned (its slots freed at once) and the branch
      makes an ordinary proposal (no new lookup);
  4b. a branch at depth d1 without a copy child looks up a copy proposal when
      no copy row outside its own ancestors is alive; if the first copied
      token passes the screen, x1 is that token (q1 one-hot) and the proposal
      opens at once as a chain of rows, each the child of the previous one,
      all at depth 0 -- they advance together, so each attends to its
      ancestors' cache rows written earlier in the same pass.  The chain is
      cut to the free table rows beyond a reserve for the ordinary tree, to
      the uncommitted window and to the token budget.  A branch whose first
      proposal is copied opens no second proposal;
  5'. verification repeats while the new root reached R in this step (chain
      rows reach R together), so one step can commit several tokens; a copied
      x1 is verified with q1 one-hot: accepted with probability p_R(x1), else
      the token is drawn from p_R with x1 removed.
A child is never created at a position that would leave the uncommitted
window (32 positions past the last committed one).
"""
from __future__ import annotations

import dataclasses
from typing import Any, Dict, List, Optional, Sequence, Tuple

import numpy as np

from . import copy as CP
from . import sampling as S

WIN = 32  # uncommitted window: a child's position minus the last committed one is < WIN


# ----------------------------------------------------------------------------
# model adapters
# ----------------------------------------------------------------------------


class OracleRows:
    """Adapter from the state machine's row calls to the fp64 LoopedModel."""

    def __init__(self, model):
        self.m = model

    def prelude(self, prefix: Sequence[int], pos: int, slots: Sequence[int]):
        return self.m.prelude(int(prefix[-1]), pos, slots)

    def iterate(self, h, r: int, prefix, pos: int, slots):
        return self.m.iterate(h, r, pos, slots)

    def readout(self, h, r: int, prefix, pos: int, slots, head: bool = True):
        hc = self.m.coda(h, r, pos, slots)
        return self.m.logits(hc) if head else None


# ----------------------------------------------------------------------------
# results
# ----------------------------------------------------------------------------


@dataclasses.dataclass
class Stats:
    steps: int = 0
    rows_sum: int = 0
    rows_max: int = 0
    n_first: int = 0
    n_second: int = 0
    n_fallback: int = 0
    gate_checks: int = 0
    gate_opens: int = 0
    branches_created: int = 0
    resid_fallback: int = 0
    table_peak: int = 0  # most branches alive at once (children exist before the same step's prune)
    copy_chains: int = 0  # copy proposals opened
    copy_rows: int = 0  # rows they opened
    copy_cut: int = 0  # copied rows pruned by the depth-d1 screen
    n_copy: int = 0  # commits of a copied token

    def gamma(self, d1: int, d2: int, R: int) -> float:
        """Mean acceptance length, Eq. 9 (section 3.2)."""
        n = self.n_first + self.n_second + self.n_fallback
        den = self.n_first * d1 + self.n_second * d2 + self.n_fallback * R
        return n * R / den if den else float("nan")


@dataclasses.dataclass
class DecodeResult:
    tokens: List[int]  # committed after the prompt: x_1 (prefill) then the decode tokens
    src: List[int]  # per decode token: 1 first proposal, 2 second, 0 full-depth draw
    commit_step: List[int]  # per decode token: step index (1-based) of its commit
    committed_slots: List[int]
    stats: Stats
    trace: List[List[Tuple[int, int, int, int]]]  # per step: (uid, slot, pos, depth) sorted by uid
    logits: Dict[Tuple[int, int], np.ndarray]  # optional readout logits keyed (pos, depth)
    step_margin: List[float] = dataclasses.field(default_factory=list)
    # per step: smallest top-1 minus top-2 probability (softmax at T = 1) over
    # the readouts whose argmax or draw that step's decisions used
    step_gap: List[float] = dataclasses.field(default_factory=list)
    # per step: smallest (z_top1 - z_top2) / max|z| over the same readouts


def top2_gap(z: np.ndarray) -> float:
    """(z_top1 - z_top2) / max|z|: how far a readout's argmax is from a tie,
    relative to the logits' scale."""
    z = np.asarray(z, np.float64)
    a = np.partition(z, -2)[-2:]
    return float((a[1] - a[0]) / np.max(np.abs(z)))


def top2_margin(z: np.ndarray) -> float:
    """p(top1) - p(top2) of softmax(z) at T = 1 (the greedy-margin reading)."""
    z = np.asarray(z, np.float64)
    p = np.exp(z - z.max())
    p /= p.sum()
    a = np.partition(p, -2)[-2:]
    return float(a[1] - a[0])


# ----------------------------------------------------------------------------
# prefill and first commit (section 2.2)
# ----------------------------------------------------------------------------


def readout_depths(R: int, d1: int, d2: int) -> List[int]:
    return sorted({r for r in (d1, d2, R) if r > 0})


def prefill(rows, prompt: Sequence[int], R: int, tags: Sequence[int],
            keep_logits: bool = False) -> Dict[Tuple[int, int], np.ndarray]:
    """Prompt positions 0..P-1 at slots 0..P-1, all depths, readouts (coda caches)
    at every depth in ``tags``.  Returns logits at (P-1, R), plus every (pos, tag)
    when ``keep_logits``."""
    P = len(prompt)
    out: Dict[Tuple[int, int], np.ndarray] = {}
    for pos in range(P):
        slots = list(range(pos + 1))
        prefix = list(prompt[:pos + 1])
        h = rows.prelude(prefix, pos, slots)
        for r in range(1, R + 1):
            h = rows.iterate(h, r, prefix, pos, slots)
            if r in tags:
                head = keep_logits or (pos == P - 1 and r == R)
                z = rows.readout(h, r, prefix, pos, slots, head=head)
                if head:
                    out[(pos, r)] = z
    return out


def first_token(z_R: np.ndarray, P: int, temperature: float, top_p: float, seed: int) -> int:
    p = S.process(z_R, temperature, top_p)
    return S.race(p, seed, P, S.AR)


# ----------------------------------------------------------------------------
# full-depth autoregressive decoding (the comparison baseline)
# ----------------------------------------------------------------------------


def decode_ar(rows, prompt: Sequence[int], R: int, max_new: int, temperature: float,
              top_p: float, seed: int, keep_logits: bool = False) -> DecodeResult:
    """Each position runs all R loops, reads out at R and commits.  The token
    at position j is drawn with the stream (j, AR)."""
    P = len(prompt)
    zs = prefill(rows, prompt, R, [R], keep_logits)
    committed = list(prompt) + [first_token(zs[(P - 1, R)], P, temperature, top_p, seed)]
    cslots = list(range(P + 1))
    st = Stats()
    logits = dict(zs) if keep_logits else {}
    src, cstep = [], []
    for _ in range(max_new):
        pos = len(committed) - 1
        slots = cslots[:pos + 1]
        h = rows.prelude(committed, pos, slots)
        for r in range(1, R + 1):
            h = rows.iterate(h, r, committed, pos, slots)
            st.steps += 1
            st.rows_sum += 1
            st.rows_max = 1
        z = rows.readout(h, R, committed, pos, slots)
        if keep_logits:
            logits[(pos, R)] = z
        p = S.process(z, temperature, top_p)
        committed.append(S.race(p, seed, pos + 1, S.AR))
        cslots.append(pos + 1)
        src.append(S.SRC_FALLBACK)
        st.n_fallback += 1
        cstep.append(st.steps)
    return DecodeResult(committed[P:], src, cstep, cslots, st, [], logits)


# ----------------------------------------------------------------------------
# pipelined speculative decoding (sections 2.2-2.4)
# ----------------------------------------------------------------------------


@dataclasses.dataclass
class Branch:
    uid: int
    parent: int
    slot: int
    pos: int  # position of the prefix's last token
    token: int  # that token
    chain: Dict[int, int]  # pos -> slot for uncommitted positions of the prefix
    depth: int = 0
    state: Any = None
    p: Optional[np.ndarray] = None  # this step's processed readout
    x1: int = -1
    q1: Optional[np.ndarray] = None
    gate: bool = False
    x2: int = -1
    q2: Optional[np.ndarray] = None
    child1: int = -1
    child2: int = -1
    # A former root left behind by an external commit: it keeps iterating and
    # taking its readouts (so its committed position gets its block and coda
    # cache rows at every depth) but decides nothing -- no proposal, no
    # verification -- is never pruned, and leaves the table once it has run
    # all R iterations.
    retiring: bool = False
    z: Optional[np.ndarray] = None  # this step's readout logits (copy screening)
    copy_row: bool = False  # its token was copied from the context
    copy_child: bool = False  # x1 is a copied token and child1 the next copy row


@dataclasses.dataclass
class CopyConfig:
    """Context-copy proposals (readings in oracle/copy.py)."""
    tau: float
    k: int = 4
    max_len: int = 16
    match_cap: int = 64
    table: int = 64  # branch-table capacity the chain must fit in
    reserve: int = 8  # rows kept free for the ordinary tree


class SpecDecoder:
    """The pipelined self-speculative decoder.  ``second``: "gated" (the method),
    "ungated" (residual second proposal always opened) or "masked" (ablation,
    section 3.4).  ``d2 = 0``: single proposal."""

    def __init__(self, rows, prompt: Sequence[int], R: int, d1: int, d2: int, max_new: int,
                 temperature: float, top_p: float, seed: int, n_slots: int,
                 second: str = "gated", keep_trace: bool = True, keep_logits: bool = False,
                 skip_prefill: bool = False, first: Optional[int] = None,
                 copy: Optional[CopyConfig] = None):
        assert 1 <= d1 < R and (d2 == 0 or d1 < d2 < R)
        self.copy = copy
        self.copy_scores: List[float] = []  # every screen score evaluated (tests check margins)
        self.rows, self.R, self.d1, self.d2 = rows, R, d1, d2
        self.T, self.top_p, self.seed = temperature, top_p, seed
        self.second = second
        self.keep_trace, self.keep_logits = keep_trace, keep_logits
        P = len(prompt)
        self.P, self.max_new = P, max_new
        self.pos_limit = P + max_new  # children only for positions < pos_limit
        self.tags = readout_depths(R, d1, d2)
        self.logits: Dict[Tuple[int, int], np.ndarray] = {}
        if skip_prefill:
            x1 = first
        else:
            zs = prefill(rows, prompt, R, self.tags, keep_logits)
            if keep_logits:
                self.logits.update(zs)
            x1 = first_token(zs[(P - 1, R)], P, temperature, top_p, seed)
        self.committed = list(prompt) + [x1]
        self.cslots = list(range(P))
        self.free = set(range(P, n_slots))
        self.branches: Dict[int, Branch] = {}
        self.next_uid = 0
        self.stats = Stats()
        self.src: List[int] = []
        self.cstep: List[int] = []
        self.trace: List[List[Tuple[int, int, int, int]]] = []
        self.step_margin: List[float] = []
        self.step_gap: List[float] = []
        root = self._new_branch(-1, P, x1, {})
        self.cslots.append(root.slot)

    # -- bookkeeping -----------------------------------------------------------
    def _alloc(self) -> int:
        if not self.free:
            raise RuntimeError("slot pool exhausted")
        s = min(self.free)
        self.free.remove(s)
        return s

    def _new_branch(self, parent: int, pos: int, token: int, chain: Dict[int, int]) -> Branch:
        b = Branch(self.next_uid, parent, self._alloc(), pos, token, dict(chain))
        b.chain[pos] = b.slot  # index copy of the parent's list + own slot (section 2.4)
        self.next_uid += 1
        self.branches[b.uid] = b
        self.stats.branches_created += 1
        self.stats.table_peak = max(self.stats.table_peak, len(self.branches))
        return b

    def slots_of(self, b: Branch) -> List[int]:
        L = len(self.committed)
        return [self.cslots[j] if j < L else b.chain[j] for j in range(b.pos + 1)]

    def prefix_of(self, b: Branch) -> List[int]:
        toks = {}
        x = b
        while x is not None:
            toks[x.pos] = x.token
            x = self.branches.get(x.parent)
        L = len(self.committed)
        return [self.committed[j] if j < L else toks[j] for j in range(b.pos + 1)]

    def root(self) -> Branch:
        L = len(self.committed)
        roots = [b for b in self.branches.values() if b.pos == L - 1]
        assert len(roots) == 1
        return roots[0]

    # -- one batched step ----------------------------------------------------------
    def step(self) -> None:
        st = self.stats
        st.steps += 1
        order = sorted(self.branches)
        rows = self.rows
        # 1. prelude for branches at depth 0
        for u in order:
            b = self.branches[u]
            if b.depth == 0:
                b.state = rows.prelude(self.prefix_of(b), b.pos, self.slots_of(b))
        # 2. one loop iteration for every branch
        for u in order:
            b = self.branches[u]
            b.state = rows.iterate(b.state, b.depth + 1, self.prefix_of(b), b.pos, self.slots_of(b))
            b.depth += 1
        st.rows_sum += len(order)
        st.rows_max = max(st.rows_max, len(order))
        if self.keep_trace:
            self.trace.append([(u, self.branches[u].slot, self.branches[u].pos,
                                self.branches[u].depth) for u in order])
        # 3. readouts
        margin = gap = float("inf")
        for u in order:
            b = self.branches[u]
            b.p = None
            if b.depth in self.tags:
                z = rows.readout(b.state, b.depth, self.prefix_of(b), b.pos, self.slots_of(b))
                if self.keep_logits:
                    self.logits[(b.pos, b.depth)] = z
                margin = min(margin, top2_margin(z))
                gap = min(gap, top2_gap(z))
                b.p = S.process(z, self.T, self.top_p)
                b.z = z
        self.step_margin.append(margin)
        self.step_gap.append(gap)
        # retiring rows that ran their last iteration leave (their slots hold
        # committed positions)
        for u in order:
            if self.branches[u].retiring and self.branches[u].depth >= self.R:
                del self.branches[u]
        # 4. proposals
        L = len(self.committed)
        for u in order:
            b = self.branches.get(u)
            if b is None or b.retiring:
                continue
            # is a child at pos+1 still needed, and inside the uncommitted window?
            spawn = b.pos + 1 < self.pos_limit and b.pos + 1 - (L - 1) < WIN
            if b.depth == self.d1:
                if b.copy_child:
                    sc = CP.screen_score(b.z, b.x1)
                    self.copy_scores.append(sc)
                    if sc >= self.copy.tau:
                        continue  # the copied token goes on
                    st.copy_cut += len(self._subtree(b.child1))
                    for v in self._subtree(b.child1):
                        self.free.add(self.branches.pop(v).slot)
                    b.child1, b.copy_child = -1, False
                    b.q1 = b.p  # an ordinary proposal; no new lookup
                    b.x1 = S.race(b.q1, self.seed, b.uid, S.PROP1)
                    if spawn:
                        b.child1 = self._new_branch(b.uid, b.pos + 1, b.x1, b.chain).uid
                    continue
                b.q1 = b.p
                b.x1 = S.race(b.q1, self.seed, b.uid, S.PROP1)
                if spawn and self.copy is not None and self._copy_allowed(b):
                    if self._open_copy(b, L):
                        continue
                if spawn:
                    b.child1 = self._new_branch(b.uid, b.pos + 1, b.x1, b.chain).uid
            elif self.d2 and b.depth == self.d2 and b.x1 >= 0 and not b.copy_child:
                st.gate_checks += 1
                if self.second == "gated":
                    b.gate = S.gate_open(b.p, b.q1, b.x1)
                    q2 = S.residual(b.p, b.q1) if b.gate else None
                elif self.second == "ungated":
                    q2 = S.residual(b.p, b.q1)
                else:
                    q2 = S.masked_second(b.p, b.x1)
                b.gate = q2 is not None
                if b.gate:
                    st.gate_opens += 1
                    b.q2 = q2
                    b.x2 = S.race(q2, self.seed, b.uid, S.PROP2)
                    if spawn:
                        b.child2 = self._new_branch(b.uid, b.pos + 1, b.x2, b.chain).uid
        # 5-6. verify at full depth, commit, prune / reroot; repeated while the
        # new root also reached R in this step (copied chains)
        while not self.done():
            root = self.root()
            if root.depth < self.R:
                return
            self._verify_commit(root)

    def _copy_allowed(self, b: Branch) -> bool:
        """No copy row alive outside b's own ancestors (b included)."""
        for x in self.branches.values():
            if x.copy_row and not x.retiring and x.uid != b.uid and b.uid not in self._subtree(x.uid):
                return False
        return True

    def _open_copy(self, b: Branch, L: int) -> bool:
        """Copy proposal for b (at depth d1, x1 already drawn): screen its first
        token and open the chain.  Returns whether a chain was opened."""
        cp = self.copy
        seq = self.prefix_of(b)
        _, _, prop = CP.lookup(seq, L, cp.k, cp.max_len, cp.match_cap)
        if not prop:
            return False
        sc = CP.screen_score(b.z, prop[0])
        self.copy_scores.append(sc)
        if sc < cp.tau:
            return False
        m = min(len(prop),
                cp.table - len(self.branches) - cp.reserve,  # free table rows beyond the reserve
                # window: the last copied row at b.pos + m stays WIN - 2 - ceil(R / d1)
                # or less past the last committed position (room for the tail's children)
                WIN - 2 - (b.pos - (L - 1)) - -(-self.R // self.d1),
                self.pos_limit - 1 - b.pos)  # token budget
        if m < 1:
            return False
        self.stats.copy_chains += 1
        self.stats.copy_rows += m
        b.x1, b.q1, b.copy_child = prop[0], S.one_hot(prop[0], len(b.p)), True
        parent = b
        for j in range(m):
            c = self._new_branch(parent.uid, parent.pos + 1, prop[j], parent.chain)
            c.copy_row = True
            if parent is b:
                b.child1 = c.uid
            else:
                parent.x1, parent.copy_child, parent.child1 = prop[j], True, c.uid
                parent.q1 = None  # set to one-hot once the row has a readout width
            parent = c
        return True

    def _verify_commit(self, root: Branch) -> None:
        st = self.stats
        q1 = S.one_hot(root.x1, len(root.p)) if root.copy_child else root.q1
        x, src, fb = S.verify(root.p, root.x1, q1, root.gate, root.x2, root.q2,
                              self.seed, root.uid)
        st.resid_fallback += fb
        self.committed.append(x)
        self.src.append(src)
        self.cstep.append(st.steps)
        if src == S.SRC_FIRST:
            st.n_first += 1
            st.n_copy += int(root.copy_child)
        elif src == S.SRC_SECOND:
            st.n_second += 1
        else:
            st.n_fallback += 1
        keep_uid = root.child1 if src == S.SRC_FIRST else root.child2 if src == S.SRC_SECOND else -1
        keep = set(self._subtree(keep_uid)) if keep_uid >= 0 else set()
        for u in sorted(self.branches):
            if u in keep or self.branches[u].retiring:
                continue
            b = self.branches.pop(u)
            if u != root.uid:  # the root's slot holds a committed position
                self.free.add(b.slot)
        if keep_uid >= 0:
            self.branches[keep_uid].parent = -1
            self.cslots.append(self.branches[keep_uid].slot)
        elif not self.done():
            L = len(self.committed)
            nr = self._new_branch(-1, L - 1, x, {})
            self.cslots.append(nr.slot)

    # -- explicit tree edits between steps ----------------------------------------
    def _subtree(self, uid: int) -> List[int]:
        out = []
        for u in sorted(self.branches):
            x = self.branches[u]
            while x is not None and x.uid != uid:
                x = self.branches.get(x.parent)
            if x is not None:
                out.append(u)
        return out

    def rollback(self, uid: int) -> None:
        """Prune branch `uid` and all its descendants (not the root); their slots
        are freed and the parent forgets the child."""
        b = self.branches[uid]
        assert uid != self.root().uid and not b.retiring
        for u in self._subtree(uid):
            self.free.add(self.branches.pop(u).slot)
        p = self.branches.get(b.parent)
        if p is not None:
            if p.child1 == uid:
                p.child1 = -1
            if p.child2 == uid:
                p.child2 = -1

    def commit_branch(self, uid: int) -> None:
        """Commit a child of the root without full-depth verification (an
        external acceptance, source 3): its token is appended, every branch
        outside its subtree is pruned and it becomes the root.  The old root
        has not run all R iterations yet, and later rows read its position's
        cache rows at every depth, so it stays in the table as a retiring row
        until it has (see Branch.retiring)."""
        root = self.root()
        b = self.branches[uid]
        assert b.parent == root.uid
        self.committed.append(b.token)
        self.src.append(3)
        self.cstep.append(self.stats.steps)
        keep = set(self._subtree(uid))
        for u in sorted(self.branches):
            x = self.branches[u]
            if u in keep or x.retiring:
                continue
            if u == root.uid:
                x.retiring = True
                x.child1 = x.child2 = x.x1 = x.x2 = -1
                x.gate = False
                x.q1 = x.q2 = None
                continue
            self.branches.pop(u)
            self.free.add(x.slot)
        b.parent = -1
        self.cslots.append(b.slot)

    def done(self) -> bool:
        return len(self.committed) >= self.P + 1 + self.max_new

    def run(self) -> DecodeResult:
        while not self.done():
            self.step()
        return DecodeResult(self.committed[self.P:], self.src, self.cstep, self.cslots,
                            self.stats, self.trace, self.logits, self.step_margin,
                            self.step_gap)


def decode_spec(rows, prompt, R, d1, d2, max_new, temperature, top_p, seed, n_slots,
                **kw) -> DecodeResult:
    return SpecDecoder(rows, prompt, R, d1, d2, max_new, temperature, top_p, seed, n_slots,
                       **kw).run()
