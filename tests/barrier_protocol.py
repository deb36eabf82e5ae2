"""A model of the mbarrier hand-offs of the tensor-core chunkwise kernel
(xlstm_mlstm_matrix_b200/csrc/chunkwise_tc.cu), and two checks on it.

Each role of the kernel (TMA producer, MMA issuer, gate warp, normaliser, state
group, token group) is written out as its sequence of barrier operations per chunk,
in program order: `wait` for a completion of a barrier, or `arrive` on it (a
tcgen05.commit or a TMA transaction counts as an arrival at the point it is
issued; the real completion can only come later).  A completion is named by the
barrier and the chunk it belongs to; a barrier with count N completes once all N
of its producers have arrived for that chunk.  The model's names: CONV_SPLIT is the
kernel's B_CONV0 (both compute groups' halves of the state split), CONV_CLO its
B_CONV1; a trailing digit is a ring slot or a pair index.

The happens-before graph has program-order edges inside a role and an edge from
every arrival of a completion to every wait for it.  Three properties are checked:

- no deadlock: the graph has no cycle, and every awaited completion gets all its
  arrivals;
- no phase overrun: for every wait on completion i of a barrier, some arrival of
  completion i+1 of the same barrier is reachable from that wait.  An mbarrier wait
  tests a phase parity, so a consumer that comes to wait for phase i after phase
  i+1 has also completed sees the parity of i again and waits for ever; the
  property says that this interleaving cannot happen, whatever the timing;
- no phase underrun: every arrival of completion i-1 reaches the op before the
  wait for completion i (the wait's start).  A consumer that skips a phase (an exact chunk's V, say) and waits
  for the next one while the skipped one is still open would see the open phase's
  parity as done.

`chunkwise_protocol(...)` writes the chunkwise kernel's protocol and
`summary_protocol(...)` that of the segment summary kernel (csrc/segments.cu).  Two earlier forms, which
the overrun check rejects: `paired=False`, one B_OPS barrier and one B_VT barrier
for two V stages; `exact_v_wait=True`, the token group waiting for an exact chunk's
V with one V stage.
"""
from __future__ import annotations

from collections import defaultdict, deque

COUNT = {"K_EMPTY": 2, "Q_EMPTY": 2, "G_EMPTY": 3, "CONV_SPLIT": 2, "KV_EMPTY": 2}


def _base(name: str) -> str:
    """The barrier kind: ring and pair barriers end in their slot digit."""
    return name.rstrip("0123456789")


class Protocol:
    def __init__(self):
        self.roles = defaultdict(list)   # role -> [(op, barrier, tag)]

    def wait(self, role, bar, tag):
        self.roles[role].append(("wait", bar, tag))

    def arrive(self, role, bar, tag):
        self.roles[role].append(("arrive", bar, tag))

    # ---- graph ------------------------------------------------------------
    def _graph(self):
        nodes, succ = [], defaultdict(list)
        arrivals, waits = defaultdict(list), defaultdict(list)
        for role, ops in self.roles.items():
            prev = None
            for i, (op, bar, tag) in enumerate(ops):
                n = (role, i)
                nodes.append(n)
                if prev is not None:
                    succ[prev].append(n)
                prev = n
                (arrivals if op == "arrive" else waits)[(bar, tag)].append(n)
        for key, ws in waits.items():
            for a in arrivals.get(key, []):
                for w in ws:
                    succ[a].append(w)
        return nodes, succ, arrivals, waits

    def check(self):
        """Returns a list of problems (empty when both properties hold)."""
        nodes, succ, arrivals, waits = self._graph()
        problems = []
        for (bar, tag), ws in waits.items():
            need = COUNT.get(_base(bar), 1)
            got = len(arrivals.get((bar, tag), []))
            if got != need:
                problems.append(f"deadlock: {bar} completion {tag} has {got} of {need} arrivals")
        # cycle check (Kahn)
        indeg = defaultdict(int)
        for n in nodes:
            for m in succ[n]:
                indeg[m] += 1
        q = deque(n for n in nodes if indeg[n] == 0)
        seen = 0
        while q:
            n = q.popleft()
            seen += 1
            for m in succ[n]:
                indeg[m] -= 1
                if indeg[m] == 0:
                    q.append(m)
        if seen != len(nodes):
            problems.append("deadlock: the happens-before graph has a cycle")
            return problems
        # phase overrun
        order = defaultdict(list)   # barrier -> completion tags in order
        for (bar, tag) in arrivals:
            order[bar].append(tag)
        for bar in order:
            order[bar].sort()
        for (bar, tag), ws in waits.items():
            tags = order.get(bar, [])
            if tag not in tags:
                continue
            i = tags.index(tag)
            if i + 1 >= len(tags):
                continue
            nxt = set(arrivals[(bar, tags[i + 1])])
            for w in ws:
                if not self._reaches(succ, w, nxt):
                    problems.append(f"overrun: {bar} completion {tags[i + 1]} can come before the wait of "
                                    f"{w[0]} for completion {tag}")
        # phase underrun: a wait for completion i must start after completion i-1 (else the
        # parity of i-1's phase, still open, already reads as i's).  The wait starts after
        # the op before it in its role; the arrivals it waits for only end it.
        for (bar, tag), ws in waits.items():
            tags = order.get(bar, [])
            if tag not in tags or tags.index(tag) == 0:
                continue
            prev = arrivals[(bar, tags[tags.index(tag) - 1])]
            for w in ws:
                start = (w[0], w[1] - 1) if w[1] > 0 else None
                if any(start is None or not self._reaches(succ, a, {start}) for a in prev):
                    problems.append(f"underrun: the wait of {w[0]} for {bar} completion {tag} can start "
                                    f"before completion {tags[tags.index(tag) - 1]}")
        return problems

    @staticmethod
    def _reaches(succ, start, targets):
        q, seen = deque([start]), {start}
        while q:
            n = q.popleft()
            if n in targets:
                return True
            for m in succ[n]:
                if m not in seen:
                    seen.add(m)
                    q.append(m)
        return False


def chunkwise_protocol(nc: int, vst: int, big: bool, exact=(), ng: int = 4, paired: bool = True,
                       exact_v_wait: bool = False) -> Protocol:
    """The hand-offs of chunk_tc_kernel for nc chunks: vst V stages (2 at L = 64, 1 at
    L = 128), big = d_qk 256 (half of C_lo through shared memory), `exact` the chunks
    that take the exact form, ng gate-ring slots.  exact_v_wait=True gives the earlier
    form in which the token group also waited for an exact chunk's V with one V stage."""
    ex = [c in set(exact) for c in range(nc)]
    P = Protocol()
    s2 = lambda name, c: f"{name}{c & 1}"                  # two-stage rings and parity pairs
    ops = (lambda c: s2("OPS", c)) if paired else (lambda c: "OPS")
    vt2 = (lambda c: s2("VT", c)) if paired else (lambda c: "VT")
    fast_rank = {}   # single-barrier B_VT: completions are numbered by fast chunks
    k = 0
    for c in range(nc):
        if not ex[c]:
            fast_rank[c] = k
            k += 1
    vt_tag = (lambda c: c) if paired else (lambda c: fast_rank[c])

    # TMA producer
    for c in range(nc):
        if c >= 2:
            P.wait("tma", s2("K_EMPTY", c), c - 2)
        P.arrive("tma", s2("K_FULL", c), c)
        if c >= 2:
            P.wait("tma", s2("Q_EMPTY", c), c - 2)
        P.arrive("tma", s2("Q_FULL", c), c)
        if vst == 1 and c >= 1:
            P.wait("tma", "V_EMPTY", c - 1)
        P.arrive("tma", s2("V_FULL", c) if vst == 2 else "V_FULL", c)

    # MMA issuer
    for c in range(nc):
        P.wait("mma", s2("K_FULL", c), c)
        P.wait("mma", s2("Q_FULL", c), c)
        if c >= 1:
            P.wait("mma", "S_EMPTY", c - 1)
        if c >= 1 and ex[c - 1]:
            P.wait("mma", "H_EMPTY", c - 1)
        P.arrive("mma", "S_FULL", c)
        P.wait("mma", f"G_FULL{c % ng}", c)
        P.wait("mma", "CONV_SPLIT", c)
        if vst == 2 and not ex[c]:
            P.wait("mma", vt2(c), vt_tag(c))
        if c >= 1 and not ex[c - 1]:
            P.wait("mma", "H_EMPTY", c - 1)
        if big:
            P.arrive("mma", "CLO_FREE", c)
            P.wait("mma", "CONV_CLO", c)
        P.wait("mma", ops(c), c)
        P.wait("mma", s2("V_FULL", c) if vst == 2 else "V_FULL", c)
        if vst == 1 and not ex[c]:
            P.wait("mma", "VT", fast_rank[c])
        P.arrive("mma", "H_FULL", c)
        P.arrive("mma", s2("Q_EMPTY", c), c)
        if ex[c]:
            P.wait("mma", "VT_EXACT", c)
        P.arrive("mma", "UPD_DONE", c)
        P.arrive("mma", s2("K_EMPTY", c), c)
        if vst == 1:
            P.arrive("mma", "V_EMPTY", c)

    # gate warp
    for c in range(nc):
        if c >= ng:
            P.wait("gate", f"G_EMPTY{c % ng}", c - ng)
        P.arrive("gate", f"G_FULL{c % ng}", c)

    # normaliser: n entering chunk c+1 goes to buffer (c+1) & 1
    P.arrive("norm", "N_READY0", 0)
    for c in range(nc):
        P.wait("norm", f"G_FULL{c % ng}", c)
        P.wait("norm", s2("K_FULL", c), c)
        if c >= 1:
            P.wait("norm", s2("N_FREE", c - 1), c - 1)
        P.arrive("norm", s2("N_READY", c + 1), c + 1)
        P.arrive("norm", s2("K_EMPTY", c), c)
        P.arrive("norm", f"G_EMPTY{c % ng}", c)

    # state group
    for c in range(nc):
        if c >= 1:
            P.wait("state", "UPD_DONE", c - 1)
        P.wait("state", f"G_FULL{c % ng}", c)
        P.arrive("state", "CONV_SPLIT", c)
        P.wait("state", s2("Q_FULL", c), c)
        P.wait("state", s2("N_READY", c), c)
        P.arrive("state", s2("Q_EMPTY", c), c)
        P.arrive("state", s2("N_FREE", c), c)
        P.wait("state", ops(c), c)
        P.wait("state", "H_FULL", c)
        if ex[c]:
            P.arrive("state", "VT_EXACT", c)
        P.arrive("state", "H_EMPTY", c)
        P.arrive("state", f"G_EMPTY{c % ng}", c)
    P.wait("state", "UPD_DONE", nc - 1)

    # token group (its loop starts at c = -1: w V(0) with two V stages)
    for c in range(-1, nc):
        if c >= 0:
            P.wait("token", f"G_FULL{c % ng}", c)
            if c >= 1:
                P.wait("token", "UPD_DONE", c - 1)
            P.arrive("token", "CONV_SPLIT", c)
            if c >= 1:
                P.wait("token", "H_FULL", c - 1)
            P.wait("token", "S_FULL", c)
            P.arrive("token", "S_EMPTY", c)
            P.arrive("token", ops(c), c)
            if vst == 2:
                P.arrive("token", f"G_EMPTY{c % ng}", c)
            else:
                if not ex[c] or exact_v_wait:
                    P.wait("token", "V_FULL", c)
                if not ex[c]:
                    P.arrive("token", "VT", fast_rank[c])
                P.arrive("token", f"G_EMPTY{c % ng}", c)
            if big:
                P.wait("token", "CLO_FREE", c)
                P.arrive("token", "CONV_CLO", c)
        if vst == 2 and c + 1 < nc:
            j = c + 1
            if c >= 0:
                P.wait("token", "CONV_SPLIT", c)
            P.wait("token", f"G_FULL{j % ng}", j)
            P.wait("token", s2("V_FULL", j), j)
            if paired or not ex[j]:
                P.arrive("token", vt2(j), vt_tag(j))
    return P


def summary_protocol(nc: int, stages: int, ring: int = 4) -> Protocol:
    """The hand-offs of the segment summary kernel (csrc/segments.cu) for nc chunks:
    `stages` k/v stages (the first `stages` copies issued before the gate scan), a
    weight ring of `ring` slots filled by two warps (even and odd chunks)."""
    P = Protocol()
    st = lambda name, c: f"{name}{c % stages}"
    wr = lambda name, c: f"{name}{c % ring}"
    # TMA producer
    for c in range(min(stages, nc)):
        P.arrive("tma", st("KV_FULL", c), c)
    for c in range(stages, nc):
        P.wait("tma", st("KV_EMPTY", c), c - stages)
        P.arrive("tma", st("KV_FULL", c), c)
    # MMA issuer
    for c in range(nc):
        P.wait("mma", st("VS", c), c)
        P.arrive("mma", st("KV_EMPTY", c), c)
    P.arrive("mma", "DONE", 0)
    # weight warps
    for w in (0, 1):
        for c in range(w, nc, 2):
            if c >= ring:
                P.wait(f"weights{w}", wr("W_EMPTY", c), c - ring)
            P.arrive(f"weights{w}", wr("W_FULL", c), c)
    # compute group: w V in place, then n_seg from k
    for c in range(nc):
        P.wait("compute", st("KV_FULL", c), c)
        P.wait("compute", wr("W_FULL", c), c)
        P.arrive("compute", st("VS", c), c)
        P.arrive("compute", wr("W_EMPTY", c), c)
        P.arrive("compute", st("KV_EMPTY", c), c)
    P.wait("compute", "DONE", 0)
    return P
