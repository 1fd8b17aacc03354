"""The barrier protocol of the prefill attention kernel (csrc/sm100_prefill.cu,
prefill_attend_kernel), modelled on the CPU.

The roles -- the TMA producer, the MMA issuer, and the four softmax warps of
each of the two query groups -- run as coroutines interleaved at random; the
tensor core completes its work in issue order (MMAs, then the commits behind
them) and the copy engine in any order.  Each mbarrier is a completion
counter whose parity waits behave as on the device.  Checked for every
interleaving drawn: no wait passes on a completion other than the one it
names (no phase aliasing), no key, value, score or P buffer is reused before
its consumer is done, each group's value GEMMs accumulate in order, and the
whole tile schedule finishes (no deadlock) -- for group lengths that differ,
that are equal, and with an empty second group.  A change to the kernel's
waits or commits must be mirrored here."""
import random

import pytest

K_STAGES = V_STAGES = 2          # key and value rings
GROUPS, WARPS = 2, 4             # query groups per CTA, softmax warps per group


class Barrier:
    def __init__(self, name, count=1):
        self.name, self.count, self.pending, self.completions = name, count, 0, 0

    def arrive(self):
        self.pending += 1
        if self.pending == self.count:
            self.pending = 0
            self.completions += 1

    def passes(self, parity):     # try_wait.parity: the phase with this parity has completed
        return (self.completions & 1) != parity


def wait(bar, parity, nth):
    """Yield until the parity wait passes; it must then have seen exactly its nth completion."""
    while not bar.passes(parity):
        yield "blocked"
    assert bar.completions == nth, f"{bar.name}: {bar.completions} completions, the wait names #{nth}"


def run_schedule(n_g, seed):
    rng = random.Random(seed)
    n_all = max(n_g)
    q_full = Barrier("q_full")
    k_full = [Barrier(f"k_full{i}") for i in range(K_STAGES)]
    k_empty = [Barrier(f"k_empty{i}") for i in range(K_STAGES)]
    v_full = [Barrier(f"v_full{i}") for i in range(V_STAGES)]
    v_empty = [Barrier(f"v_empty{i}") for i in range(V_STAGES)]
    s_full = [[Barrier(f"s_full{g}{b}") for b in range(2)] for g in range(GROUPS)]
    s_free = [[Barrier(f"s_free{g}{b}", WARPS) for b in range(2)] for g in range(GROUPS)]
    p_full = [Barrier(f"p_full{g}", WARPS) for g in range(GROUPS)]
    o_done = [[Barrier(f"o_done{g}{b}") for b in range(2)] for g in range(GROUPS)]
    tensor_queue, copies = [], []                    # tensor core in order; copies in any order
    k_tile, v_tile = [None] * K_STAGES, [None] * V_STAGES
    s_tile = [[None, None] for _ in range(GROUPS)]   # tile held by each score buffer
    p_tile = [None] * GROUPS                          # tile held by each group's P buffer
    o_last = [-1] * GROUPS                            # last value GEMM accumulated per group

    def producer():
        copies.append((q_full, None, None))
        for i in range(n_all):
            if i >= K_STAGES:
                yield from wait(k_empty[i % K_STAGES], ((i // K_STAGES) - 1) & 1, i // K_STAGES)
            copies.append((k_full[i % K_STAGES], ("k", i % K_STAGES), i))
            yield "step"
            if i >= V_STAGES:
                yield from wait(v_empty[i % V_STAGES], ((i // V_STAGES) - 1) & 1, i // V_STAGES)
            copies.append((v_full[i % V_STAGES], ("v", i % V_STAGES), i))
            yield "step"

    def issuer():
        yield from wait(q_full, 0, 1)

        def value_gemms(t):
            sv = t % V_STAGES
            yield from wait(v_full[sv], (t // V_STAGES) & 1, t // V_STAGES + 1)
            for g in range(GROUPS):
                if t >= n_g[g]:
                    continue
                yield from wait(p_full[g], t & 1, t + 1)
                tensor_queue.append(("O", g, t, sv))
                tensor_queue.append(("commit", o_done[g][t & 1]))
                yield "step"
            tensor_queue.append(("commit", v_empty[sv]))

        for i in range(n_all):
            sk, sb = i % K_STAGES, i & 1
            yield from wait(k_full[sk], (i // K_STAGES) & 1, i // K_STAGES + 1)
            for g in range(GROUPS):
                if i >= n_g[g]:
                    continue
                if i >= 2:
                    yield from wait(s_free[g][sb], ((i >> 1) - 1) & 1, i >> 1)
                tensor_queue.append(("S", g, i, sk))
                tensor_queue.append(("commit", s_full[g][sb]))
                yield "step"
            tensor_queue.append(("commit", k_empty[sk]))
            if i >= 1:
                yield from value_gemms(i - 1)
        yield from value_gemms(n_all - 1)

    def softmax(g, warp):
        for i in range(n_g[g]):
            sb = i & 1
            yield from wait(s_full[g][sb], (i >> 1) & 1, (i >> 1) + 1)
            assert s_tile[g][sb] == i
            if i >= 1:                                # O and the P tile are free
                yield from wait(o_done[g][(i - 1) & 1], ((i - 1) >> 1) & 1, ((i - 1) >> 1) + 1)
                assert o_last[g] == i - 1
            yield "step"
            assert s_tile[g][sb] == i, "score buffer overwritten before the second read"
            if warp == 0:
                p_tile[g] = i
            s_free[g][sb].arrive()
            p_full[g].arrive()
            yield "step"
        if n_g[g]:
            last = n_g[g] - 1
            yield from wait(o_done[g][last & 1], (last >> 1) & 1, (last >> 1) + 1)
            assert o_last[g] == last

    roles = {"producer": producer(), "issuer": issuer()}
    roles.update({f"softmax{g}{w}": softmax(g, w) for g in range(GROUPS) for w in range(WARPS)})
    finished, idle = set(), 0
    while len(finished) < len(roles):
        who = rng.choice([r for r in roles if r not in finished] + ["tensor", "copy"])
        progressed = False
        if who == "tensor":
            if tensor_queue:
                op = tensor_queue.pop(0)
                progressed = True
                if op[0] == "S":
                    _, g, i, sk = op
                    assert k_tile[sk] == i, "key tile replaced before its score GEMM"
                    s_tile[g][i & 1] = i
                elif op[0] == "O":
                    _, g, t, sv = op
                    assert v_tile[sv] == t and p_tile[g] == t, "value or P tile replaced too early"
                    assert o_last[g] == t - 1
                    o_last[g] = t
                else:
                    op[1].arrive()
        elif who == "copy":
            if copies:
                bar, slot, tile = copies.pop(rng.randrange(len(copies)))
                progressed = True
                if slot is not None:
                    (k_tile if slot[0] == "k" else v_tile)[slot[1]] = tile
                bar.arrive()
        else:
            try:
                progressed = next(roles[who]) != "blocked"
            except StopIteration:
                finished.add(who)
                progressed = True
        idle = 0 if progressed else idle + 1
        assert idle < 20000, f"deadlock with group lengths {n_g}"


@pytest.mark.parametrize("n_g", [(1, 1), (1, 0), (2, 0), (1, 3), (2, 4), (3, 5), (8, 8), (30, 32)])
def test_prefill_barrier_protocol(n_g):
    for seed in range(12):
        run_schedule(n_g, seed * 13 + sum(n_g))
