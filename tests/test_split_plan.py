"""Invariants of the decode kernel's automatic split, restated on the host.

The partition kernel plans the automatic split on the device: each
(request, KV head) group is padded to 32-token quanta (an empty request to
one) behind two empty cost quanta, the groups are laid end to end, and warp w
takes the w-th of Weff equal slices of that line.  A group cut by slices is
merged by a tree of merge nodes of fan-in 8 (d = 128) or 16 (d = 64).  The
kernel relies on these facts, checked here over many batches:

- every token quantum of every group lies in exactly one piece, and every
  piece holds at least one token (an empty request: exactly one piece);
- the pieces of a group number at most ceil(max_len / 128) + 1, the bound the
  workspace is sized for;
- a warp holds at most two pieces of split groups (its first and its last),
  so two shared-memory slots hold the first-level merge nodes it completes;
- split indices run 0..n-1 within a group, and the merge tree's slot and
  counter indices are distinct and inside the workspace's row and counter
  region.

This is host logic (integer scheduling), not the oracle: no attention
arithmetic is involved.
"""
import numpy as np
import pytest

QUANTUM, COST, MIN_SHARE = 32, 2, 128


def cdiv(a, b):
    return -(-a // b)


def max_pieces(max_len):
    return cdiv(max(max_len, 1), MIN_SHARE) + 1


def tree_slots(n, fan):
    total = n
    while n > fan:
        n = cdiv(n, fan)
        total += n
    return total


def tree_nodes(n, fan):
    total = 0
    while n > 1:
        n = cdiv(n, fan)
        total += n
    return total


def plan(lens, hkv, warps):
    """Pieces (warp, group, first token, tokens, split index, splits)."""
    groups = []  # (start quantum, token quanta, length)
    at = 0
    for L in lens:
        real = max(1, cdiv(L, QUANTUM))
        for _ in range(hkv):
            groups.append((at, real, L))
            at += COST + real
    total = at
    weff = min(warps, max(1, total // (MIN_SHARE // QUANTUM)))
    start = lambda w: w * total // weff  # noqa: E731
    slice_of = lambda x: ((x + 1) * weff - 1) // total  # noqa: E731
    pieces = []
    gi = 0
    for w in range(weff):
        a, b = start(w), start(w + 1)
        while gi < len(groups) and groups[gi][0] + COST + groups[gi][1] <= a:
            gi += 1
        k = gi
        while k < len(groups) and groups[k][0] < b:
            g0, real, L = groups[k]
            first, end = g0 + COST, g0 + COST + real
            lo, hi = max(a, first), min(b, end)
            if hi > lo:
                t0 = (lo - first) * QUANTUM
                ntok = max(0, min((hi - first) * QUANTUM, L) - t0)
                n = slice_of(end - 1) - slice_of(first) + 1
                pieces.append((w, k, t0, ntok, w - slice_of(first), n))
            k += 1
    return groups, pieces, weff


def check(lens, hkv, warps, fan):
    groups, pieces, weff = plan(lens, hkv, warps)
    bound = max_pieces(max(lens) if len(lens) else 1)
    slots, nodes = tree_slots(bound, fan), tree_nodes(bound, fan)
    by_group = {}
    for w, k, t0, ntok, s, n in pieces:
        by_group.setdefault(k, []).append((t0, ntok, s, n, w))
    assert sorted(by_group) == list(range(len(groups))), "a group got no piece"
    for k, ps in by_group.items():
        L = groups[k][2]
        ps.sort()
        n = ps[0][3]
        assert all(p[3] == n for p in ps) and len(ps) == n, "piece count disagrees with nsplit"
        assert sorted(p[2] for p in ps) == list(range(n)), "split indices are not 0..n-1"
        assert n <= bound, f"{n} pieces > workspace bound {bound}"
        if L == 0:
            assert n == 1 and ps[0][1] == 0
            continue
        covered = 0
        for t0, ntok, _, _, _ in ps:
            assert t0 == covered and ntok > 0, "pieces must tile the tokens in order"
            covered += ntok
        assert covered == L
        # merge tree: slots of pieces and inner nodes, counters of all nodes
        if n > 1:
            seen_slots, seen_ctr = set(range(n)), set()
            level, off = n, 0
            while level > 1:
                up, offup = cdiv(level, fan), off + level
                for jp in range(up):
                    c = offup - n + jp
                    assert c not in seen_ctr and 0 <= c < nodes
                    seen_ctr.add(c)
                    if up > 1:
                        slot = offup + jp
                        assert slot not in seen_slots and slot < slots
                        seen_slots.add(slot)
                level, off = up, offup
            assert len(seen_ctr) == tree_nodes(n, fan)
    split_pieces = {}
    for w, k, *_ in pieces:
        if by_group[k][0][3] > 1:
            split_pieces[w] = split_pieces.get(w, 0) + 1
    assert max(split_pieces.values(), default=0) <= 2, "a warp holds more than two split pieces"
    return len(pieces), weff


WARPS = [148 * 12, 148 * 8, 132 * 12, 7]


@pytest.mark.parametrize("warps", WARPS)
def test_benchmark_shapes(warps):
    rng = np.random.default_rng(11)
    shapes = [
        (rng.integers(128, 4097, 64), 8, 8),                                 # Qwen3-shaped decode batch
        (np.array([32768, 65536, 98304, 131072]), 8, 16),                    # long contexts, d = 64
        (np.clip(np.round(np.exp(np.log(1536) + 0.8 * rng.standard_normal(256))), 16, 16384).astype(int), 8, 8),
        (rng.integers(256, 4097, 56), 8, 8),                                 # decode rows of the mixed batch
        (np.array([7, 33, 64, 100]), 8, 8),                                  # tiny
    ]
    for lens, hkv, fan in shapes:
        check([int(x) for x in lens], hkv, warps, fan)


@pytest.mark.parametrize("seed", range(40))
def test_random_batches(seed):
    rng = np.random.default_rng(seed)
    B = int(rng.integers(1, 300))
    kind = seed % 4
    if kind == 0:
        lens = rng.integers(0, 5000, B)
    elif kind == 1:
        lens = np.where(rng.random(B) < 0.3, 0, rng.integers(1, 70, B))   # many empty and tiny
    elif kind == 2:
        lens = rng.integers(1, 200000, max(1, B // 50))                     # few, very long
    else:
        lens = np.clip(np.round(np.exp(6 + 1.5 * rng.standard_normal(B))), 0, 60000)
    hkv = int(rng.choice([1, 2, 4, 8]))
    warps = int(rng.choice(WARPS))
    fan = int(rng.choice([8, 16]))
    check([int(x) for x in lens], hkv, warps, fan)


def test_edge_batches():
    for lens in ([0], [1], [0, 0, 0], [31, 32, 33], [1] * 500, [128] * 3, [200000]):
        for warps in (1, 2, 1776):
            check(lens, 1, warps, 8)
            check(lens, 8, warps, 16)
