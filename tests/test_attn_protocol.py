"""A randomised model of the attention kernel's mbarrier protocol.

The kernel's warps meet only at mbarriers and at the tensor pipe, so the
protocol can be checked on the CPU: this model runs the MMA issuer's fixed
issue order, every softmax warp (with valid rows or not), the TMA producer, the tail
warps' stage releases and an in-order tensor pipe whose commit arrives once
every earlier MMA has run, in random interleavings. It checks:

  * every parity wait polls only while its barrier has completed k or k + 1
    phases, k being the phase it waits for (otherwise the parity is
    ambiguous);
  * a softmax warp reads scores S_n while their buffer still holds them;
    PV_n runs after every warp with valid rows stored P_n; new scores are
    written into a buffer only after the PV that reads its P ran;
  * O_t is rescaled at tile j after PV_t(j-1) ran and before PV_t(j) runs;
  * a K/V stage is reloaded only after every MMA reading it ran;
  * nothing deadlocks.

The schedule modelled is the kernel's: score tile n = j * nq + t goes to
TMEM buffer n % NB (NB = 3 for head_dim 64 with two query tiles, else 2) with
its P stored over it; per-buffer s_full / p_full barriers; the issuer issues
S_0 .. S_{NB-1}, then PV_n (once P_n is written) followed by S_{n+NB} (once
its K/V tile has landed), for n = 0, 1, ...; a softmax warp waits for
PV_t(j-1) only when it rescales O_t. The negative tests drop one rule each
and find the failure it prevents.

A model is not the kernel: it checks the protocol's logic only.
"""
import random

import pytest

ST = 4   # K/V stages


class Violation(Exception):
    pass


class Bar:
    def __init__(self, name, count):
        self.name, self.count, self.done, self.pend = name, count, 0, 0

    def arrive(self, n=1):
        for _ in range(n):
            self.pend += 1
            if self.pend == self.count:
                self.done += 1
                self.pend = 0

    def test(self, k, who):
        """Parity test for the completion of phase k."""
        if not (k <= self.done <= k + 1):
            raise Violation(f"{who} waits for phase {k} of {self.name}, {self.done} completed")
        return self.done == k + 1


def run(nq, n_tiles, active, tail, seed, nb=None, gate_slack=0, idle_warps_wait=True, rescale_p=0.2):
    """nb: S/P buffers (default: the kernel's choice, 3 for two query tiles
    else 2). gate_slack: NB - gate_slack scores are issued before the first
    PV, so S_n follows PV_{n-NB+gate_slack} (0 is the kernel's rule, -1 one
    PV too early). idle_warps_wait: warps without valid rows wait for
    their scores before they arrive (the kernel's rule)."""
    rng = random.Random(seed)
    if nb is None:
        nb = 3 if nq == 2 else 2
    s_full = [Bar(f"s_full{b}", 1) for b in range(3)]
    p_full = [Bar(f"p_full{b}", 128) for b in range(3)]
    pv_done = [Bar(f"pv_done{t}", 1) for t in range(2)]
    kv_full = [Bar(f"kv_full{s}", 1) for s in range(ST)]
    kv_empty = [Bar(f"kv_empty{s}", 1 + (2 if tail else 0)) for s in range(ST)]
    o_final = Bar("o_final", 1)
    pipe, ran, holds, p_written, stage = [], set(), {}, {}, {}
    n_all = n_tiles * nq

    def execute(op):
        if op[0] == "commit":
            op[1].arrive()
            return
        kind, n = op
        j, t, b = n // nq, n % nq, n % nb
        if stage.get(j % ST) != j:
            raise Violation(f"{kind}_{n} runs without its K/V tile")
        if kind == "S":
            if n >= nb and ("PV", n - nb) not in ran:
                raise Violation(f"S_{n} overwrites buffer {b} before PV_{n - nb} read its P")
            holds[b] = n
        else:
            if holds.get(b) != n:
                raise Violation(f"PV_{n} reads buffer {b} holding S_{holds.get(b)}")
            if p_written.get(n, set()) != {w for w in range(4) if active[t][w]}:
                raise Violation(f"PV_{n} runs before P_{n} is written")
        ran.add((kind, n))

    def issuer():
        # the kernel's fixed order: S_0 .. S_{NB-1}, then PV_n and S_{n+NB}
        # for n = 0, 1, ...; each op blocks on its own barrier
        prefill = min(nb - gate_slack, n_all)
        st = {"ns": 0, "np": 0, "kv": -1, "after_pv": False, "done": False}

        def issue_s():
            ns = st["ns"]
            j = ns // nq
            if j > st["kv"]:
                if not kv_full[j % ST].test(j // ST, "issuer"):
                    return False
                st["kv"] = j
            pipe.append(("S", ns))
            pipe.append(("commit", s_full[ns % nb]))
            st["ns"] = ns + 1
            return True

        def step():
            if st["done"]:
                return None
            if st["ns"] < prefill:
                return issue_s()
            if st["after_pv"]:
                if st["ns"] < n_all and not issue_s():
                    return False
                st["after_pv"] = False
                return True
            np_ = st["np"]
            if np_ == n_all:
                pipe.append(("commit", o_final))
                st["done"] = True
                return True
            if not p_full[np_ % nb].test(np_ // nb, "issuer"):
                return False
            pipe.append(("PV", np_))
            pipe.append(("commit", pv_done[np_ % nq]))
            if np_ % nq == nq - 1:   # every MMA of K/V tile np_ // nq issued
                pipe.append(("commit", kv_empty[(np_ // nq) % ST]))
            st["np"] = np_ + 1
            st["after_pv"] = True
            return True
        return step

    def softmax_warp(t, w):
        rows = active[t][w]
        st = {"j": 0, "pc": 0, "rescale": False}
        who = f"softmax {t}.{w}"

        def step():
            j, pc = st["j"], st["pc"]
            if j >= n_tiles:
                if pc == 0:
                    if not o_final.test(0, who):
                        return False
                    st["pc"] = 1
                    return True
                return None
            n = j * nq + t
            b = n % nb
            if pc == 0:                           # S_n computed
                if rows or idle_warps_wait:
                    if not s_full[b].test(n // nb, who):
                        return False
                st["pc"] = 1 if rows else 5
            elif pc == 1:                         # first half of the scores read
                if holds.get(b) != n:
                    raise Violation(f"{who} reads S_{n}, buffer {b} holds {holds.get(b)}")
                st["pc"] = 2
            elif pc == 2:                         # second half read; P stored over the first
                if holds.get(b) != n:
                    raise Violation(f"{who} reads S_{n}, buffer {b} holds {holds.get(b)}")
                st["rescale"] = j > 0 and rng.random() < rescale_p
                st["pc"] = 3
            elif pc == 3:                         # O rescale: wait for PV_t(j-1) only then
                if st["rescale"]:
                    if not pv_done[t].test(j - 1, who):
                        return False
                    if ("PV", n - nq) not in ran or ("PV", n) in ran:
                        raise Violation(f"{who} rescales O_{t} at tile {j} while a PV may run")
                st["pc"] = 4
            elif pc == 4:                         # P stores complete
                p_written.setdefault(n, set()).add(w)
                st["pc"] = 5
            elif pc == 5:                         # P_n handed over
                p_full[b].arrive(32)
                st["j"], st["pc"] = j + 1, 0
            return True
        return step

    def producer():
        st = {"j": 0}

        def step():
            j = st["j"]
            if j >= n_tiles:
                return None
            if j >= ST:
                if not kv_empty[j % ST].test(j // ST - 1, "producer"):
                    return False
                for n in range((j - ST) * nq, (j - ST + 1) * nq):
                    for kind in ("S", "PV"):
                        if (kind, n) not in ran:
                            raise Violation(f"stage reloaded before {kind}_{n} ran")
            stage[j % ST] = j
            kv_full[j % ST].arrive()
            st["j"] = j + 1
            return True
        return step

    def tail_warp():
        st = {"j": 0}

        def step():
            j = st["j"]
            if j >= n_tiles:
                return None
            if not kv_full[j % ST].test(j // ST, "tail"):
                return False
            kv_empty[j % ST].arrive()
            st["j"] = j + 1
            return True
        return step

    def tensor_pipe():
        if not pipe:
            return False
        execute(pipe.pop(0))
        return True

    actors = [issuer(), producer()]
    actors += [softmax_warp(t, w) for t in range(nq) for w in range(4)]
    actors += [tail_warp(), tail_warp()] if tail else []
    finished = [False] * len(actors)
    while True:
        if all(finished) and not pipe:
            return
        order = list(range(len(actors) + 1))
        rng.shuffle(order)
        moved = False
        for i in order:
            if i == len(actors):
                moved = tensor_pipe()
            elif not finished[i]:
                r = actors[i]()
                if r is None:
                    finished[i] = True
                moved = bool(r)
            if moved:
                break
        if not moved and not all(finished):
            raise Violation("deadlock")


def random_case(seed, nq=None):
    rng = random.Random(seed)
    nq = nq or rng.choice([1, 2])
    active = [[True] * 4 for _ in range(2)]
    if rng.random() < 0.5:   # a short frame: some warps have no valid rows
        active = [[True] + [rng.random() < 0.5 for _ in range(3)] for _ in range(2)]
    return dict(nq=nq, n_tiles=rng.randint(1, 10), active=active,
                tail=nq == 2 and rng.random() < 0.5, seed=seed)


def violations(cases, nq=None, **rules):
    found = []
    for seed in range(cases):
        try:
            run(**random_case(seed, nq), **rules)
        except Violation as e:
            found.append((seed, str(e)))
    return found


@pytest.mark.parametrize("nq", [1, 2])
def test_kernel_schedule_is_race_free(nq):
    assert violations(1500, nq=nq) == []


def test_two_buffers_with_two_query_tiles_are_race_free():
    """The head_dim 128 kernel: two buffers, so S_t(j+1) follows PV_t(j)."""
    assert violations(800, nq=2, nb=2) == []


def test_scores_issued_one_pv_early_overwrite_p():
    """S_n issued once PV_{n-NB-1} is issued (one PV too early) can
    overwrite P_{n-NB} before the PV that reads it has run."""
    found = violations(300, gate_slack=-1, rescale_p=0.0)
    assert any("overwrites" in msg for _, msg in found)


def test_three_buffers_with_one_query_tile_break_the_rescale_wait():
    """With one query tile and three buffers, S_t(j) completing no longer
    implies PV_t(j-2) completed, so the O rescale's parity wait on pv_done
    can see the phase before the one it waits for."""
    found = violations(400, nq=1, nb=3, rescale_p=0.5)
    assert any("pv_done" in msg for _, msg in found)


def test_idle_warps_must_wait_for_their_scores():
    """p_full counts arrivals: warps without valid rows that arrive without
    waiting for S_n run ahead and complete a phase before the warps with
    rows have written P."""
    found = violations(300, idle_warps_wait=False)
    assert found
    assert all(random_case(seed)["active"] != [[True] * 4] * 2 for seed, _ in found)
